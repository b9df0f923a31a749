// Host-side check of the library's bit-level helpers, compiled and run by
// tests/test_device_helpers.py: the order-preserving keys of the routers' warp
// top-k (order_key / key_value), the bf16 conversions and the scaled e4m3
// widening of the FP8 and FP4 GEMMs. Reads float32 bit patterns from a file, writes the
// helpers' results to another (and the widening of all 256 codes to a third).
// No device code runs.
#include <stdio.h>
#include <stdlib.h>

#include "../sparse_moe_transformer_gemm_b200/csrc/common.cuh"

int main(int argc, char** argv) {
    if (argc != 3 && argc != 4) return 2;
    if (argc == 4) {
        // the FP8 GEMM's scaled e4m3 widening: codes i (low half) and 255 - i
        FILE* e8 = fopen(argv[3], "wb");
        if (!e8) return 1;
        for (uint32_t i = 0; i < 256; ++i) {
            const uint32_t r = moe::e4m3_pair_scaled_bits((255u - i) << 24 | i << 8);
            fwrite(&r, sizeof r, 1, e8);
        }
        // the FP4 GEMM's scaled E2M1 widening: byte i (two codes)
        for (uint32_t i = 0; i < 256; ++i) {
            const uint32_t r = moe::e2m1_pair_scaled_bits(i);
            fwrite(&r, sizeof r, 1, e8);
        }
        if (fclose(e8) != 0) return 1;
    }
    FILE* in = fopen(argv[1], "rb");
    FILE* out = fopen(argv[2], "wb");
    if (!in || !out) return 1;
    uint32_t u;
    while (fread(&u, sizeof u, 1, in) == 1) {
        const float f = moe::f32_from_bits(u);
        const uint32_t key = moe::order_key(f);
        const float back = moe::key_value(key);
        const uint16_t b = moe::float_to_bf16_bits(f);
        const float2 w = moe::bf16x2_to_float2(moe::pack_bf16x2(f, -f));
        const uint32_t rec[5] = {key, moe::f32_bits(back), b, moe::f32_bits(w.x),
                                 moe::f32_bits(w.y)};
        fwrite(rec, sizeof rec, 1, out);
    }
    fclose(in);
    return fclose(out) == 0 ? 0 : 1;
}
