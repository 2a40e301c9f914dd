// fc_gemm.cu -- persistent grouped GEMM for FC1 (+SwiGLU) and FC2 with MXFP4
// weights on the 5th-generation tensor cores (tcgen05, accumulators in TMEM).
//
// What it computes (tokenspeed-situ package description, intro: "FC1 MXFP4 +
// <gated activation>" and the matching FC2; b12x package description, "What's
// in here": "W4A16 ... with inline FP4 weight dequant"): for every row block
// (an expert's slice of at most 128 grouped rows) and every 256-row tile of
// that expert's weight,
//     D[rows, 256] = A[rows, K] . W[256, K]^T,   f32 accumulation,
// with W decoded from MXFP4 (E2M1 code * 2^(E8M0 - 127)) to bf16 on chip.
// FC1 tiles pair 128 gate rows with the matching 128 up rows, so the epilogue
// applies h = silu(gate) * up in registers (and, on the w4a8 path, the MXFP8
// round trip of h: tokenspeed-situ package description, "Activation precision
// (w4a16 vs w4a8)").
//
// Per CTA (one per SM, persistent over work units u = (row block, tile)):
//   warp 0      producer: TMA of the activation tile (128 x 64 bf16, 128-byte
//               swizzle) and of the FP4 weight tile (256 x 32 bytes), cp.async
//               of the scale bytes; one mbarrier per stage.
//   warps 2-5   dequant: FP4 + E8M0 -> bf16 into the 128-byte swizzled
//               K-major layout the tensor core reads.
//   warp 1      MMA issuer (one thread) + TMEM owner; tcgen05.mma kind::f16,
//               commits free the stage and publish the accumulator.
//   warps 6-9   epilogue: tcgen05.ld -> FC1: SwiGLU -> bf16 stores,
//               FC2: f32 stores (the combine rounds once, at the end); the
//               accumulator is double-buffered in TMEM (2 x 256 columns).
// Orientation per work unit: a block of more than `swap_rows` rows runs with
// tokens on the MMA's M side (M = 128, N = 256 weight rows); a smaller block
// (decode) runs weight rows on M (two M = 128 MMAs, gate/up or lower/upper
// half) and its tokens on N (16..128), so the tensor core does not multiply
// padding rows.  Every wait is bounded; a wait that gives up records an error
// word and the CTA drains its own copies and MMAs before freeing TMEM.
#include "kernels.cuh"
#include "ptx.cuh"

namespace moe_mx {

namespace {

constexpr int kStages = 3;
constexpr int kThreads = 320;
constexpr int kActBytes = 128 * 128;      // 128 rows x 64 bf16
constexpr int kWbBytes = 256 * 128;       // 256 rows x 64 bf16 (dequantised)
constexpr int kFp4Bytes = 256 * 32;       // 256 rows x 64 FP4 codes
constexpr int kSclBytes = 256 * 4;        // 256 rows x one 4-byte scale word
constexpr int kOffAct = 0;
constexpr int kOffWb = kOffAct + kStages * kActBytes;
constexpr int kOffFp4 = kOffWb + kStages * kWbBytes;
constexpr int kOffScl = kOffFp4 + kStages * kFp4Bytes;
constexpr int kOffBar = kOffScl + kStages * kSclBytes;
constexpr int kNumBars = 4 * kStages + 4 + 1;
constexpr int kOffTmemSlot = kOffBar + kNumBars * 8;
constexpr int kSmemBytes = kOffTmemSlot + 16 + 1024; // + slack for 1024-byte alignment
constexpr uint32_t kTmemCols = 512;
constexpr unsigned long long kDrainTimeoutNs = 200000000ull; // 0.2 s for the final drains

struct Bars {
    uint32_t base;
    __device__ uint32_t full_tma(int s) const { return base + 8 * s; }
    __device__ uint32_t full_deq(int s) const { return base + 8 * (kStages + s); }
    __device__ uint32_t empty(int s) const { return base + 8 * (2 * kStages + s); }
    __device__ uint32_t mma_done() const { return base + 8 * (3 * kStages); }
    __device__ uint32_t acc_full(int b) const { return base + 8 * (3 * kStages + 1 + b); }
    __device__ uint32_t acc_empty(int b) const { return base + 8 * (3 * kStages + 3 + b); }
};

__device__ __forceinline__ float silu_mul(float g, float u)
{
    return g / (1.0f + expf(-g)) * u;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&v);
}

// Store 32 floats as bf16 (64 contiguous bytes).
__device__ __forceinline__ void store_bf16x32(__nv_bfloat16 *dst, const float (&v)[32])
{
    uint4 *d = reinterpret_cast<uint4 *>(dst);
#pragma unroll
    for (int i = 0; i < 4; ++i)
        d[i] = make_uint4(pack_bf16x2(v[8 * i + 0], v[8 * i + 1]), pack_bf16x2(v[8 * i + 2], v[8 * i + 3]),
                          pack_bf16x2(v[8 * i + 4], v[8 * i + 5]), pack_bf16x2(v[8 * i + 6], v[8 * i + 7]));
}

// MXFP8 round trip of 32 values held by one thread (quantise, then dequantise).
__device__ __forceinline__ void mxfp8_roundtrip32(float (&v)[32])
{
    uint8_t c[32];
    const uint32_t sb = mx_quantize32_e4m3(v, c);
    const float scale = (sb == 0xFF) ? __uint_as_float(0x7FC00000u) : exp2_int((int)sb - 127);
#pragma unroll
    for (int i = 0; i < 32; ++i)
        v[i] = __fmul_rn(e4m3_to_f32(c[i]), scale);
}

// MXFP8 round trip of one value per lane, the 32 lanes forming one MX block.
__device__ __forceinline__ float mxfp8_roundtrip_warp(float v)
{
    float amax = fabsf(v);
    bool finite = amax <= 3.402823466e38f;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
        amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, off));
    finite = __all_sync(0xFFFFFFFFu, finite);
    if (!finite)
        return __uint_as_float(0x7FC00000u);
    int s = (amax == 0.f) ? -127 : floor_log2_pos(amax) - 8;
    s = max(-127, min(127, s));
    const uint32_t code = f32_to_e4m3(__fmul_rn(v, exp2_int(-s)));
    return __fmul_rn(e4m3_to_f32(code), exp2_int(s));
}

} // namespace

__global__ void __launch_bounds__(kThreads, 1)
    fc_gemm_kernel(const FcGemmArgs a, const __grid_constant__ CUtensorMap act_map,
                   const __grid_constant__ CUtensorMap w_map)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *const gsm = smem_raw + (base - raw); // generic pointer to the aligned base
    const Bars bars{base + kOffBar};
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(bars.full_tma(s), 1 + 32); // producer's expect_tx + 32 cp.async arrivals
            mbar_init(bars.full_deq(s), 128);    // every dequant thread
            mbar_init(bars.empty(s), 1);         // MMA commit
        }
        mbar_init(bars.mma_done(), 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(bars.acc_full(b), 1);   // MMA commit
            mbar_init(bars.acc_empty(b), 128); // every epilogue thread
        }
        fence_mbar_init();
        fence_proxy_async_smem();
        prefetch_tensormap(&act_map);
        prefetch_tensormap(&w_map);
    }
    if (warp == 1) {
        tmem_alloc(base + kOffTmemSlot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t *>(gsm + kOffTmemSlot);

    const int nrb = *a.num_rowblocks;
    const int total_units = nrb * a.n_tiles;
    const int kst = a.K / 64;
    const int half_rows = a.fc1 ? a.R / 2 : 0; // FC1: offset of the up rows
    const unsigned long long tmo = a.timeout_ns;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        uint32_t g = 0;
        bool ok = true;
        const int scl_ld = a.K / 32;
        for (int u = blockIdx.x; ok && u < total_units; u += gridDim.x) {
            const int4 blk = a.rowblocks[u / a.n_tiles];
            const int nt = u % a.n_tiles;
            const int wrow_a = blk.x * a.R + (a.fc1 ? nt * 128 : nt * 256);
            const int wrow_b = a.fc1 ? wrow_a + half_rows : wrow_a + 128;
            for (int kk = 0; kk < kst; ++kk, ++g) {
                const int s = g % kStages;
                const uint32_t ph = (g / kStages) & 1;
                bool w = true;
                if (lane == 0)
                    w = mbar_wait_bounded(bars.empty(s), ph ^ 1, a.err, tmo);
                w = __shfl_sync(0xFFFFFFFFu, w, 0);
                if (!w) {
                    ok = false;
                    break;
                }
                const uint32_t scl = base + kOffScl + s * kSclBytes;
                for (int r = lane; r < 256; r += 32) {
                    const int wr = r < 128 ? wrow_a + r : wrow_b + (r - 128);
                    cp_async_4(scl + 4 * r, a.wscale + (size_t)wr * scl_ld + (kk >> 1) * 4);
                }
                cp_async_mbar_arrive_noinc(bars.full_tma(s));
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive_expect_tx(bars.full_tma(s), kActBytes + kFp4Bytes);
                    tma_load_2d(base + kOffAct + s * kActBytes, &act_map, kk * 64, blk.y, bars.full_tma(s));
                    const uint32_t f = base + kOffFp4 + s * kFp4Bytes;
                    tma_load_2d(f, &w_map, kk * 32, wrow_a, bars.full_tma(s));
                    tma_load_2d(f + kFp4Bytes / 2, &w_map, kk * 32, wrow_b, bars.full_tma(s));
                }
                __syncwarp();
            }
        }
        // drain: every stage issued must have landed before the CTA may exit
        if (lane == 0) {
            const uint32_t first = g > (uint32_t)kStages ? g - kStages : 0u;
            for (uint32_t q = first; q < g; ++q)
                mbar_wait_bounded(bars.full_tma(q % kStages), (q / kStages) & 1, nullptr, kDrainTimeoutNs);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            uint32_t g = 0, cnt = 0;
            bool ok = true;
            for (int u = blockIdx.x; ok && u < total_units; u += gridDim.x, ++cnt) {
                const int4 blk = a.rowblocks[u / a.n_tiles];
                const bool swap = blk.z <= a.swap_rows;
                const uint32_t npad = (uint32_t)((blk.z + 15) & ~15);
                const uint32_t idesc = swap ? idesc_bf16_f32(128, npad) : idesc_bf16_f32(128, 256);
                const int buf = cnt & 1;
                if (!mbar_wait_bounded(bars.acc_empty(buf), ((cnt >> 1) & 1) ^ 1, a.err, tmo)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d = tmem_base + buf * 256;
                for (int kk = 0; kk < kst; ++kk, ++g) {
                    const int s = g % kStages;
                    const uint32_t ph = (g / kStages) & 1;
                    if (!mbar_wait_bounded(bars.full_tma(s), ph, a.err, tmo) ||
                        !mbar_wait_bounded(bars.full_deq(s), ph, a.err, tmo)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t act = base + kOffAct + s * kActBytes;
                    const uint32_t wb = base + kOffWb + s * kWbBytes;
#pragma unroll
                    for (int k16 = 0; k16 < 4; ++k16) {
                        const uint64_t da = smem_desc_sw128(act + 32 * k16);
                        const uint64_t dw = smem_desc_sw128(wb + 32 * k16);
                        const uint32_t acc = (kk | k16) != 0;
                        if (!swap) {
                            umma_f16_ss(d, da, dw, idesc, acc);
                        } else {
                            const uint64_t dw_hi = smem_desc_sw128(wb + kWbBytes / 2 + 32 * k16);
                            umma_f16_ss(d, dw, da, idesc, acc);
                            umma_f16_ss(d + 128, dw_hi, da, idesc, acc);
                        }
                    }
                    umma_commit(bars.empty(s));
                }
                if (ok)
                    umma_commit(bars.acc_full(buf));
            }
            // all MMAs must have completed before TMEM is released
            umma_commit(bars.mma_done());
            mbar_wait_bounded(bars.mma_done(), 0, nullptr, kDrainTimeoutNs);
        }
        __syncwarp();
    } else if (warp >= 2 && warp < 6) {
        // ------------------------------------------------------------ dequant
        const int t = threadIdx.x - 64; // 0..127
        uint32_t g = 0;
        bool ok = true;
        for (int u = blockIdx.x; ok && u < total_units; u += gridDim.x) {
            for (int kk = 0; kk < kst; ++kk, ++g) {
                const int s = g % kStages;
                const uint32_t ph = (g / kStages) & 1;
                if (!mbar_wait_bounded(bars.full_tma(s), ph, a.err, tmo)) {
                    ok = false;
                    break;
                }
                const uint8_t *fp4 = gsm + kOffFp4 + s * kFp4Bytes;
                const uint8_t *scl = gsm + kOffScl + s * kSclBytes;
                uint8_t *wb = gsm + kOffWb + s * kWbBytes;
                const int sh = (kk & 1) * 16;
#pragma unroll
                for (int rr = 0; rr < 2; ++rr) {
                    const int r = t + 128 * rr;
                    const uint4 q0 = *reinterpret_cast<const uint4 *>(fp4 + r * 32);
                    const uint4 q1 = *reinterpret_cast<const uint4 *>(fp4 + r * 32 + 16);
                    const uint32_t sw = *reinterpret_cast<const uint32_t *>(scl + r * 4);
                    const uint32_t sb0 = (sw >> sh) & 0xFF, sb1 = (sw >> (sh + 8)) & 0xFF;
                    const uint32_t words[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const uint32_t wv = words[c];
                        const uint32_t sb = c < 4 ? sb0 : sb1;
                        uint32_t o[4];
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const uint32_t byte = (wv >> (8 * j)) & 0xFF;
                            o[j] = e2m1_bf16_bits(byte & 0xF, sb) | (e2m1_bf16_bits(byte >> 4, sb) << 16);
                        }
                        *reinterpret_cast<uint4 *>(wb + r * 128 + ((c ^ (r & 7)) << 4)) =
                            make_uint4(o[0], o[1], o[2], o[3]);
                    }
                }
                fence_proxy_async_smem();
                mbar_arrive(bars.full_deq(s));
            }
        }
    } else if (warp >= 6) {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3; // TMEM lane quarter this warp may access
        uint32_t cnt = 0;
        for (int u = blockIdx.x; u < total_units; u += gridDim.x, ++cnt) {
            const int4 blk = a.rowblocks[u / a.n_tiles];
            const int nt = u % a.n_tiles;
            const int rows = blk.z;
            const bool swap = rows <= a.swap_rows;
            const int buf = cnt & 1;
            if (!mbar_wait_bounded(bars.acc_full(buf), (cnt >> 1) & 1, a.err, tmo))
                break;
            tc_fence_after();
            const uint32_t tb = tmem_base + ((uint32_t)(32 * q) << 16) + buf * 256;
            if (!swap) {
                const int rl = 32 * q + lane;
                const bool valid = rl < rows;
                if (a.fc1) {
                    __nv_bfloat16 *orow = static_cast<__nv_bfloat16 *>(a.out) + (size_t)(blk.y + rl) * a.out_ld;
                    for (int c = 0; c < 4; ++c) {
                        uint32_t g0[16], g1[16], u0[16], u1[16];
                        tmem_ld16(tb + 32 * c, g0);
                        tmem_ld16(tb + 32 * c + 16, g1);
                        tmem_ld16(tb + 128 + 32 * c, u0);
                        tmem_ld16(tb + 128 + 32 * c + 16, u1);
                        tmem_wait_ld();
                        float h[32];
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            h[i] = silu_mul(__uint_as_float(g0[i]), __uint_as_float(u0[i]));
                            h[16 + i] = silu_mul(__uint_as_float(g1[i]), __uint_as_float(u1[i]));
                        }
                        if (a.act_mxfp8)
                            mxfp8_roundtrip32(h);
                        if (valid)
                            store_bf16x32(orow + nt * 128 + 32 * c, h);
                    }
                } else {
                    float *orow = static_cast<float *>(a.out) + (size_t)(blk.y + rl) * a.out_ld + nt * 256;
                    for (int c = 0; c < 16; ++c) {
                        uint32_t y0[16];
                        tmem_ld16(tb + 16 * c, y0);
                        tmem_wait_ld();
                        if (valid) {
                            uint4 *d = reinterpret_cast<uint4 *>(orow + 16 * c);
#pragma unroll
                            for (int i = 0; i < 4; ++i)
                                d[i] = make_uint4(y0[4 * i], y0[4 * i + 1], y0[4 * i + 2], y0[4 * i + 3]);
                        }
                    }
                }
            } else {
                const int L = 32 * q + lane; // weight row within the 128-row half
                const int npad = (rows + 15) & ~15;
                for (int n0 = 0; n0 < npad; n0 += 16) {
                    uint32_t v0[16], v1[16];
                    tmem_ld16(tb + n0, v0);
                    tmem_ld16(tb + 128 + n0, v1);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const int n = n0 + j;
                        if (n >= rows)
                            break;
                        if (a.fc1) {
                            __nv_bfloat16 *orow = static_cast<__nv_bfloat16 *>(a.out) + (size_t)(blk.y + n) * a.out_ld;
                            float hv = silu_mul(__uint_as_float(v0[j]), __uint_as_float(v1[j]));
                            if (a.act_mxfp8)
                                hv = mxfp8_roundtrip_warp(hv);
                            orow[nt * 128 + L] = __float2bfloat16_rn(hv);
                        } else {
                            float *orow = static_cast<float *>(a.out) + (size_t)(blk.y + n) * a.out_ld;
                            orow[nt * 256 + L] = __uint_as_float(v0[j]);
                            orow[nt * 256 + 128 + L] = __uint_as_float(v1[j]);
                        }
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(bars.acc_empty(buf));
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

size_t fc_gemm_smem_bytes() { return (size_t)kSmemBytes; }

cudaError_t fc_gemm_prepare()
{
    return cudaFuncSetAttribute(fc_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
}

void launch_fc_gemm(const FcGemmArgs &a, const CUtensorMap &act_map, const CUtensorMap &w_map, int grid,
                    cudaStream_t s)
{
    fc_gemm_kernel<<<grid, kThreads, kSmemBytes, s>>>(a, act_map, w_map);
}

// ---------------------------------------------------------------- watchdog self-test
// Waits on a flag that nothing sets; the bounded wait gives up, records the
// timeout in the error word, and the kernel returns normally.
__global__ void watchdog_kernel(uint32_t *err, unsigned long long timeout_ns)
{
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);
        fence_mbar_init();
        mbar_wait_bounded(smem_u32(&bar), 0, err, timeout_ns); // records kErrTimeout in *err
    }
}

void launch_watchdog(uint32_t *err, unsigned long long timeout_ns, cudaStream_t s)
{
    watchdog_kernel<<<1, 32, 0, s>>>(err, timeout_ns);
}

} // namespace moe_mx
