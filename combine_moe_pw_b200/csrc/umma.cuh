// umma.cuh - tcgen05 (5th-generation tensor core) helpers for sm_100a:
// shared-memory matrix descriptors, the kind::f16 instruction descriptor,
// TMEM allocation, MMA issue/commit, TMEM loads and 2-D TMA tile loads.
//
// Descriptor bit layouts follow the PTX ISA's tcgen05 "shared memory matrix
// descriptor" and "instruction descriptor" formats; a host test checks these
// encoders bit for bit against CUTLASS's cute::UMMA descriptor unions.
#pragma once

#include <cstdint>

namespace moe_pw {
namespace umma {

// Shared-memory matrix descriptor (64 bits):
//   [0,14)  start address >> 4      [16,30) leading byte offset >> 4
//   [32,46) stride byte offset >> 4 [46,48) version (1 on sm_100)
//   [49,52) base offset             [52]    LBO mode
//   [61,64) layout: 0 none, 1 128B-base32B, 2 128B, 4 64B, 6 32B swizzle
__host__ __device__ __forceinline__ uint64_t smem_desc(uint32_t smem_addr, uint32_t lbo_bytes,
                                                       uint32_t sbo_bytes, uint32_t layout,
                                                       uint32_t base_offset = 0)
{
    uint64_t d = 0;
    d |= uint64_t((smem_addr >> 4) & 0x3FFFu);
    d |= uint64_t((lbo_bytes >> 4) & 0x3FFFu) << 16;
    d |= uint64_t((sbo_bytes >> 4) & 0x3FFFu) << 32;
    d |= uint64_t(1u) << 46;
    d |= uint64_t(base_offset & 0x7u) << 49;
    d |= uint64_t(layout & 0x7u) << 61;
    return d;
}

constexpr uint32_t LAYOUT_SWIZZLE_128B = 2;

// Instruction descriptor for kind::f16 (32 bits):
//   [4,6) D format (1 = f32)   [7,10) A format (0 f16, 1 bf16)
//   [10,13) B format           [15] A major (0 = K)  [16] B major (0 = K)
//   [17,23) N >> 3             [24,29) M >> 4
__host__ __device__ __forceinline__ uint32_t idesc_f16(uint32_t M, uint32_t N, bool bf16,
                                                       bool a_mn_major = false,
                                                       bool b_mn_major = false)
{
    const uint32_t fmt = bf16 ? 1u : 0u;
    uint32_t d = 0;
    d |= 1u << 4;               // f32 accumulator
    d |= fmt << 7;              // A
    d |= fmt << 10;             // B (same type as A: kind::f16 does not mix)
    d |= (a_mn_major ? 1u : 0u) << 15;
    d |= (b_mn_major ? 1u : 0u) << 16;
    d |= ((N >> 3) & 0x3Fu) << 17;
    d |= ((M >> 4) & 0x1Fu) << 24;
    return d;
}

__device__ __forceinline__ void tmem_alloc(uint32_t *smem_dst, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst))),
                 "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish()
{
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void fence_before_sync()
{
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void fence_after_sync()
{
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, one M x N x 16 step issued by one thread.
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                         uint32_t idesc, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive once on `bar` when every tcgen05 op this thread issued so far is done.
__device__ __forceinline__ void commit(uint64_t *bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     static_cast<uint32_t>(__cvta_generic_to_shared(bar)))
                 : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread i gets lane (quarter*32 + i).
// The load and its wait sit in one asm block, so no use of v can be scheduled
// before the registers are valid.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
          "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
          "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]),
          "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]),
          "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
        : "r"(taddr)
        : "memory");
}

// 2-D tiled TMA load into this CTA's shared memory, completion on `bar`.
// c0 is the inner (contiguous) coordinate in elements.
__device__ __forceinline__ void tma_load_2d(void *dst, const void *tmap, int32_t c0, int32_t c1,
                                            uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
        "l"(tmap), "r"(c0), "r"(c1),
        "r"(static_cast<uint32_t>(__cvta_generic_to_shared(bar)))
        : "memory");
}

// The same load with an L2 eviction policy (createpolicy) for the tile.
__device__ __forceinline__ void tma_load_2d_hint(void *dst, const void *tmap, int32_t c0,
                                                 int32_t c1, uint64_t *bar, uint64_t policy)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
        "l"(tmap), "r"(c0), "r"(c1), "r"(static_cast<uint32_t>(__cvta_generic_to_shared(bar))),
        "l"(policy)
        : "memory");
}

// ---------------------------------------------------------------------------
// Pairs of CTAs (a cluster of 2 on neighbouring SMs) sharing one MMA:
// tcgen05 ops with .cta_group::2.  The even CTA (rank 0) issues the MMAs;
// each CTA supplies half of A's rows and half of B's rows from its own shared
// memory (same offsets), and each CTA's TMEM receives the accumulator rows of
// its half of A.
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint32_t cluster_ctarank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ uint32_t cluster_id_x()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
    return r;
}

__device__ __forceinline__ uint32_t cluster_count_x()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
    return r;
}

// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t smem_addr, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr), "r"(rank));
    return r;
}

// Every thread of both CTAs (divergent arrival allowed).
__device__ __forceinline__ void cluster_sync()
{
    asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}

// Arrive on an mbarrier given by its cluster address (this or the peer CTA).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr)
{
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
                 : "memory");
}

// Issued by one warp of each CTA of the pair; both get the same TMEM address.
__device__ __forceinline__ void tmem_alloc_pair(uint32_t *smem_dst, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst))),
                 "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish_pair()
{
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

// D (+)= A * B^T over the pair: M = 256 (128 rows from each CTA), N split in
// halves between the CTAs' B tiles.  Issued by one thread of the even CTA.
__device__ __forceinline__ void mma_bf16_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                              uint32_t idesc, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive once on `bar` in both CTAs of the pair (same shared-memory offset;
// CTA mask 0b11) when the pair MMAs issued so far are done.  This is the
// tcgen05.commit form with a CTA mask; it signals barriers only and moves
// no data.
__device__ __forceinline__ void commit_pair_both(uint64_t *bar)
{
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
        " [%0], %1;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(bar))),
        "h"(static_cast<unsigned short>(3))
        : "memory");
}

// 2-D tiled TMA load into this CTA's shared memory whose completion is
// counted on an mbarrier of either CTA of the pair (cluster address).
__device__ __forceinline__ void tma_load_2d_pair(void *dst, const void *tmap, int32_t c0,
                                                 int32_t c1, uint32_t mbar_cluster_addr,
                                                 uint64_t policy)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        ".L2::cache_hint [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(
            static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
        "l"(tmap), "r"(c0), "r"(c1), "r"(mbar_cluster_addr), "l"(policy)
        : "memory");
}

}  // namespace umma
}  // namespace moe_pw
