// Host-only check: this library's tcgen05 descriptor encoders against
// CUTLASS's cute::UMMA descriptor unions (compiled as host code, no GPU).
#include <cstdio>
#include <cute/arch/mma_sm100_desc.hpp>
#include <cute/numeric/numeric_types.hpp>
#include "umma.cuh"

int main()
{
    int bad = 0;
    const uint32_t addrs[] = {0u, 1024u, 49152u, 196608u + 1024u, 0x3FFF0u, 32u, 64u, 96u};
    for (uint32_t a : addrs)
        for (uint32_t sbo : {1024u, 512u, 2048u})
            for (uint32_t lbo : {16u, 0u, 4096u}) {
                cute::UMMA::SmemDescriptor d;
                d.start_address_ = uint16_t(a >> 4);
                d.leading_byte_offset_ = uint16_t(lbo >> 4);
                d.stride_byte_offset_ = uint16_t(sbo >> 4);
                d.version_ = 1;
                d.base_offset_ = 0;
                d.lbo_mode_ = 0;
                d.layout_type_ = uint8_t(cute::UMMA::LayoutType::SWIZZLE_128B);
                const uint64_t mine = moe_pw::umma::smem_desc(a, lbo, sbo, moe_pw::umma::LAYOUT_SWIZZLE_128B);
                if (uint64_t(d) != mine) {
                    std::printf("smem desc mismatch a=%u lbo=%u sbo=%u: %llx vs %llx\n", a, lbo, sbo,
                                (unsigned long long)uint64_t(d), (unsigned long long)mine);
                    ++bad;
                }
            }
    for (uint32_t M : {64u, 128u, 256u})
        for (uint32_t N : {16u, 64u, 128u, 256u})
            for (int bf : {0, 1}) {
                cute::UMMA::InstrDescriptor i;
                i.desc_ = 0;
                i.c_format_ = 1;
                i.a_format_ = bf;
                i.b_format_ = bf;
                i.a_major_ = 0;
                i.b_major_ = 0;
                i.n_dim_ = N >> 3;
                i.m_dim_ = M >> 4;
                const uint32_t mine = moe_pw::umma::idesc_f16(M, N, bf != 0);
                if (uint32_t(i) != mine) {
                    std::printf("idesc mismatch M=%u N=%u bf16=%d: %x vs %x\n", M, N, bf,
                                uint32_t(i), mine);
                    ++bad;
                }
            }
    // the two shapes the kernels issue, against CUTLASS's own constructor
    // (M = 256 is the two-SM form: 128 rows from each CTA of the pair)
    {
        using namespace cute;
        const uint32_t ref128 = uint32_t(UMMA::make_instr_desc<bfloat16_t, bfloat16_t, float, 128, 256,
                                                               UMMA::Major::K, UMMA::Major::K>());
        const uint32_t ref256 = uint32_t(UMMA::make_instr_desc<bfloat16_t, bfloat16_t, float, 256, 256,
                                                               UMMA::Major::K, UMMA::Major::K>());
        if (ref128 != moe_pw::umma::idesc_f16(128, 256, true) ||
            ref256 != moe_pw::umma::idesc_f16(256, 256, true)) {
            std::printf("make_instr_desc mismatch: %x %x\n", ref128, ref256);
            ++bad;
        }
    }
    std::printf(bad ? "FAIL %d\n" : "OK\n", bad);
    return bad != 0;
}
