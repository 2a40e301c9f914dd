// kernels.cuh -- constants, argument structs and launchers shared by the
// library's translation units.  Internal to libmoe_mx.so.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "ptx.cuh"

namespace moe_mx {

constexpr int kMaxExperts = 1024;
constexpr int kMaxTopK = 32;
constexpr int kBlockRows = 128;   // grouped-layout segment granularity = GEMM row block
constexpr int kRouteChunk = 64;   // tokens per router CTA (= per histogram chunk)
constexpr int kRouteThreads = 512;

struct RouteGroupArgs {
    const float *logits;
    int T, E, k;
    int32_t *topk_ids;
    float *topk_w;
    int32_t *chunk_hist;
    int32_t *counts;
    int32_t *pad_offsets;
    int4 *rowblocks;
    int32_t *num_rowblocks;
    int32_t *sorted_pair;
    int32_t *pos_of_pair;
};

void launch_route_and_group(const RouteGroupArgs &a, cudaStream_t s);
void launch_gather(const __nv_bfloat16 *x, int P, int H, int k, const int32_t *pos_of_pair, __nv_bfloat16 *A,
                   int act_mxfp8, int num_sms, cudaStream_t s);
void launch_combine(const float *Y, int T, int H, int k, const int32_t *pos_of_pair, const float *topk_w,
                    __nv_bfloat16 *out, int num_sms, cudaStream_t s);
void launch_mx_quantize(const float *src, int64_t rows, int64_t K, int fmt, uint8_t *codes, uint8_t *scales,
                        int num_sms, cudaStream_t s);

// Grouped FC GEMM (FC1 with SwiGLU, or FC2) over the row-block list.
struct FcGemmArgs {
    const int4 *rowblocks;       // {expert, first grouped row, rows, 0}
    const int32_t *num_rowblocks;
    const uint8_t *wscale;       // E8M0 scales of the weight, [E*R, K/32]
    void *out;                   // FC1: bf16 Hbuf [rows, I]; FC2: f32 Y [rows, H]
    uint32_t *err;
    unsigned long long timeout_ns;
    int K;                       // reduction length (FC1: H, FC2: I)
    int R;                       // weight rows per expert (FC1: 2I, FC2: H)
    int n_tiles;                 // 256-row weight tiles per expert (FC1: I/128, FC2: H/256)
    int out_ld;                  // leading dimension of out (FC1: I, FC2: H)
    int fc1;                     // 1: gate/up rows + SwiGLU epilogue
    int act_mxfp8;               // FC1 only: MXFP8 round trip of h before it is stored
    int swap_rows;               // row blocks of at most this many rows (<= 128) put the
                                 // weight rows on the MMA M side and the tokens on N
};

void launch_fc_gemm(const FcGemmArgs &a, const CUtensorMap &act_map, const CUtensorMap &w_map, int grid,
                    cudaStream_t s);
size_t fc_gemm_smem_bytes();
cudaError_t fc_gemm_prepare();

void launch_watchdog(uint32_t *err, unsigned long long timeout_ns, cudaStream_t s);

// ---------------------------------------------------------------- MX device helpers
// Quantise 32 values to MXFP8 E4M3 with the shared-scale rule of the OCP MX
// specification (s = floor(log2 amax) - 8, clamped to [-127, 127]); returns the
// scale byte and writes the 32 codes.
__device__ __forceinline__ uint32_t mx_quantize32_e4m3(const float (&v)[32], uint8_t (&codes)[32])
{
    float amax = 0.f;
    bool finite = true;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        const float a = fabsf(v[i]);
        finite = finite && (a <= 3.402823466e38f);
        amax = fmaxf(amax, a);
    }
    if (!finite) {
#pragma unroll
        for (int i = 0; i < 32; ++i)
            codes[i] = 0;
        return 0xFF;
    }
    int s = (amax == 0.f) ? -127 : floor_log2_pos(amax) - 8;
    s = max(-127, min(127, s));
    const float inv = exp2_int(-s);
#pragma unroll
    for (int i = 0; i < 32; ++i)
        codes[i] = (uint8_t)f32_to_e4m3(__fmul_rn(v[i], inv));
    return (uint32_t)(s + 127);
}

// MXFP8 round trip of 32 bf16 values held in four uint4: quantise, then write
// back the exact dequantised values (E4M3 value * 2^s is representable in bf16).
__device__ __forceinline__ void mxfp8_roundtrip_bf16x32(uint4 (&v)[4])
{
    float f[32];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&v[i]);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float2 t = __bfloat1622float2(h2[j]);
            f[8 * i + 2 * j] = t.x;
            f[8 * i + 2 * j + 1] = t.y;
        }
    }
    uint8_t c[32];
    const uint32_t sb = mx_quantize32_e4m3(f, c);
    const float scale = (sb == 0xFF) ? __uint_as_float(0x7FC00000u) : exp2_int((int)sb - 127);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        __nv_bfloat162 *h2 = reinterpret_cast<__nv_bfloat162 *>(&v[i]);
#pragma unroll
        for (int j = 0; j < 4; ++j)
            h2[j] = __floats2bfloat162_rn(__fmul_rn(e4m3_to_f32(c[8 * i + 2 * j]), scale),
                                          __fmul_rn(e4m3_to_f32(c[8 * i + 2 * j + 1]), scale));
    }
}

} // namespace moe_mx
