// Prints the library's tcgen05 descriptors for a set of arguments (host-side
// evaluation of the same encoder functions the kernels call), one per line:
//   <name> <argument...> <value>
// Read by tests/test_descriptors.py, which checks every field against the
// descriptor tables of the PTX ISA.
#include <cstdint>
#include <cstdio>
#include "ptx.cuh"
#include "ptx_bs.cuh"

using namespace fp8bs;

int main()
{
    const uint32_t addrs[] = {0u, 32u, 1024u, 0x12340u, 0x1B000u, 0x30000u, 0x3FFF0u};
    for (uint32_t a : addrs) {
        std::printf("smem_desc_k_sw128 %u %llu\n", a, (unsigned long long)smem_desc_k_sw128(a));
        std::printf("smem_desc_mn_sw64 %u %llu\n", a, (unsigned long long)smem_desc_mn_sw64(a));
        std::printf("smem_desc_mn_sw128 %u %llu\n", a, (unsigned long long)smem_desc_mn_sw128(a, 16384u));
        std::printf("smem_desc_cp_rows16 %u %llu\n", a, (unsigned long long)smem_desc_cp_rows16(a));
    }
    const uint32_t shapes[][2] = {{128, 256}, {128, 128}, {128, 64}, {256, 128}, {256, 256}, {64, 8}};
    for (const auto& s : shapes) {
        std::printf("idesc_e4m3_f32 %u %u %u\n", s[0], s[1], idesc_e4m3_f32(s[0], s[1]));
        for (uint32_t b = 0; b < 2; ++b)
            std::printf("idesc_e4m3_f32_major %u %u %u %u\n", s[0], s[1], b, idesc_e4m3_f32_major(s[0], s[1], b));
        for (uint32_t id = 0; id < 4; ++id)
            std::printf("idesc_e4m3_bs %u %u %u %u\n", s[0], s[1], id, idesc_e4m3_bs(s[0], s[1], id));
    }
    return 0;
}
