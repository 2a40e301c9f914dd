// quant.cu -- MX quantisation of float32 rows on the GPU (OCP Microscaling
// Formats v1.0: per 32-element block, shared scale exponent
// s = floor(log2(amax)) - emax_elem clamped to [-127, 127], stored as the E8M0
// byte s + 127; elements rounded to nearest-even onto the element grid,
// saturating; a block holding a NaN or an infinity gets scale byte 0xFF and zero
// codes).  Used to prepare MXFP4 weights.  The MXFP8 path runs mx_encode32, the
// encoder the forward's gather and FC1 epilogue run on activations.
#include "kernels.cuh"
#include "ptx.cuh"

namespace moe_mx {

namespace {

__device__ __forceinline__ uint32_t mx_quantize32_e2m1(const float (&v)[32], uint8_t (&packed)[16])
{
    float amax = 0.f;
    bool finite = true;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        const float a = fabsf(v[i]);
        finite = finite && (a <= kMaxFinite);
        amax = fmaxf(amax, a);
    }
    if (!finite) {
#pragma unroll
        for (int i = 0; i < 16; ++i)
            packed[i] = 0;
        return 0xFF;
    }
    int s = (amax == 0.f) ? -127 : floor_log2_pos(amax) - 2;
    s = max(-127, min(127, s));
    const float inv = exp2_int(-s);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const uint32_t lo = f32_to_e2m1(__fmul_rn(v[2 * i], inv));
        const uint32_t hi = f32_to_e2m1(__fmul_rn(v[2 * i + 1], inv));
        packed[i] = (uint8_t)(lo | (hi << 4));
    }
    return (uint32_t)(s + 127);
}

__global__ void __launch_bounds__(256) mx_quantize_kernel(const float *__restrict__ src, long long nblocks, int fmt,
                                                          uint8_t *__restrict__ codes, uint8_t *__restrict__ scales)
{
    for (long long b = blockIdx.x * (long long)blockDim.x + threadIdx.x; b < nblocks;
         b += (long long)gridDim.x * blockDim.x) {
        float v[32];
        const float4 *s4 = reinterpret_cast<const float4 *>(src + b * 32);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float4 f = __ldg(s4 + i);
            v[4 * i] = f.x;
            v[4 * i + 1] = f.y;
            v[4 * i + 2] = f.z;
            v[4 * i + 3] = f.w;
        }
        if (fmt == 0) {
            uint8_t p[16];
            scales[b] = (uint8_t)mx_quantize32_e2m1(v, p);
            uint4 o;
            uint8_t *ob = reinterpret_cast<uint8_t *>(&o);
#pragma unroll
            for (int i = 0; i < 16; ++i)
                ob[i] = p[i];
            reinterpret_cast<uint4 *>(codes)[b] = o;
        } else {
            uint32_t c[8], unused[8];
            uint32_t s0, s1;
            mx_encode32(v, 1, c, unused, s0, s1);
            scales[b] = (uint8_t)s0;
            store_codes32(codes + 32 * b, c);
        }
    }
}

} // namespace

void launch_mx_quantize(const float *src, int64_t rows, int64_t K, int fmt, uint8_t *codes, uint8_t *scales,
                        int num_sms, cudaStream_t s)
{
    const long long nblocks = (long long)rows * (K / 32);
    const long long want = (nblocks + 255) / 256;
    const long long cap = (long long)num_sms * 16;
    const int grid = (int)(want < cap ? want : cap);
    mx_quantize_kernel<<<grid > 0 ? grid : 1, 256, 0, s>>>(src, nblocks, fmt, codes, scales);
}

// ---------------------------------------------------------------- activation encoders (test entry)
// Encode float32 rows [rows, K] into the activation operand format with the encoders the
// forward runs: method 0 = store_act_block32 (one thread per 32-element block: the gather, which
// encodes bf16 values, and the FC1 epilogue of units with the tokens on M), method 1 =
// store_act_warp32 (one warp per block: the FC1 epilogue of units with the tokens on N).
__global__ void __launch_bounds__(256) encode_act_kernel(const float *__restrict__ src, int rows, int K, int act_mxfp8,
                                                         int method, uint8_t *__restrict__ q, uint8_t *__restrict__ sf)
{
    const long long nblocks = (long long)rows * (K / 32);
    const long long gid = blockIdx.x * (long long)blockDim.x + threadIdx.x;
    const long long stride = (long long)gridDim.x * blockDim.x;
    if (method == 0) {
        for (long long b = gid; b < nblocks; b += stride) {
            const int row = (int)(b / (K / 32)), col = (int)(b % (K / 32)) * 32;
            float v[32];
            const float4 *s4 = reinterpret_cast<const float4 *>(src + (size_t)row * K + col);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float4 f = __ldg(s4 + i);
                v[4 * i] = f.x;
                v[4 * i + 1] = f.y;
                v[4 * i + 2] = f.z;
                v[4 * i + 3] = f.w;
            }
            store_act_block32(q, sf, rows, K, row, col, v, act_mxfp8);
        }
    } else {
        const int lane = threadIdx.x & 31;
        for (long long wb = gid >> 5; wb < nblocks; wb += stride >> 5) { // warp-uniform
            const int row = (int)(wb / (K / 32)), col = (int)(wb % (K / 32)) * 32 + lane;
            store_act_warp32(q, sf, rows, K, row, col, __ldg(src + (size_t)row * K + col), act_mxfp8, lane);
        }
    }
}

void launch_encode_act(const float *src, int rows, int K, int act_mxfp8, int method, uint8_t *q, uint8_t *sf,
                       int num_sms, cudaStream_t s)
{
    const long long threads = (long long)rows * (K / 32) * (method == 0 ? 1 : 32);
    const long long want = (threads + 255) / 256;
    const int grid = (int)(want < (long long)num_sms * 16 ? want : (long long)num_sms * 16);
    encode_act_kernel<<<grid > 0 ? grid : 1, 256, 0, s>>>(src, rows, K, act_mxfp8, method, q, sf);
}

// ---------------------------------------------------------------- scale tiling
// One thread per (atom, tile row): 4 scale bytes (the 4 blocks of one K stage) in, 4 out.
__global__ void __launch_bounds__(256) tile_scales_kernel(const uint8_t *__restrict__ src, uint8_t *__restrict__ dst,
                                                          long long n_items, int R, int K, int fc1)
{
    const int kst = K / 128, ld = K / 32;
    const int n_tiles = R / 128; // FC1: I/64 tiles of 64 gate + 64 up rows (R = 2I); FC2: H/128
    for (long long it = blockIdx.x * (long long)blockDim.x + threadIdx.x; it < n_items;
         it += (long long)gridDim.x * blockDim.x) {
        const int m = (int)(it & 127);
        const long long atom = it >> 7; // ((e * n_tiles + nt) * kst + kk)
        const int kk = (int)(atom % kst);
        const long long et = atom / kst;
        const int nt = (int)(et % n_tiles);
        const long long e = et / n_tiles;
        const int row = fc1 ? (m < 64 ? nt * 64 + m : R / 2 + nt * 64 + (m - 64)) : nt * 128 + m;
        const uint32_t v = *reinterpret_cast<const uint32_t *>(src + (e * R + row) * (long long)ld + kk * 4);
        *reinterpret_cast<uint32_t *>(dst + atom * 512 + sf_atom_offset(m, 0)) = v;
    }
}

void launch_tile_scales(const uint8_t *src, uint8_t *dst, int E, int R, int K, int fc1, int num_sms, cudaStream_t s)
{
    const long long n_items = (long long)E * (R / 128) * (K / 128) * 128;
    const long long want = (n_items + 255) / 256;
    const int grid = (int)(want < (long long)num_sms * 16 ? want : (long long)num_sms * 16);
    tile_scales_kernel<<<grid > 0 ? grid : 1, 256, 0, s>>>(src, dst, n_items, R, K, fc1);
}

} // namespace moe_mx
