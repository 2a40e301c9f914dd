// kernels.cuh -- constants, argument structs and launchers shared by the
// library's translation units.  Internal to libmoe_mx.so.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "ptx.cuh"

namespace moe_mx {

// Launch `kernel` on `s`; with pdl, as a programmatic dependent of the kernel before it in the
// stream (it may start early: everything it reads from that kernel comes after grid_dep_wait).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_kernel(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                                 bool pdl, Args &&...args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

constexpr int kMaxExperts = 1024;
constexpr int kMaxTopK = 32;
constexpr int kBlockRows = 128;   // grouped-layout segment granularity = GEMM row block
constexpr int kRouteChunk = 64;   // tokens per router CTA (= per histogram chunk)
constexpr int kRouteThreads = 1024; // 32 warps: two tokens of a 64-token chunk per warp
constexpr int kSmallRouteTokens = 64; // at most this many tokens: routing and grouping in one CTA

struct RouteGroupArgs {
    const float *logits;   // [T, E - n_shared]: the routed experts' logits
    int T, E, k;           // E, k: expert slots and slots per token, shared ones included
    int32_t *topk_ids;
    float *topk_w;
    int32_t *chunk_hist;
    int32_t *counts;
    int32_t *pad_offsets;
    int4 *rowblocks;
    int32_t *num_rowblocks;
    int32_t *sorted_pair;
    int32_t *pos_of_pair;
    int split_rows; // rows per work block of the row-block list: 16, 32, 64 or kBlockRows
    int32_t *unit_counters; // optional: the GEMMs' 2 work-unit counters, zeroed here
    // Routing given instead of computed (logits unused): global expert ids [T, k] and their
    // weights; ids in [id_offset, id_offset + E) are this shard's local experts, any other id
    // is left out of the grouping (local id -1, pos_of_pair -1).
    const int32_t *given_ids = nullptr;
    const float *given_w = nullptr;
    int id_offset = 0;
    // Shared expert: its n_shared chunks are expert slots E - n_shared.., and every token's
    // last n_shared slots route to them with weight 1 (the router picks k - n_shared routed
    // experts among the first E - n_shared).  Logits form only.
    int n_shared = 0;
    // Logits form over a shard: the router picks among route_E experts (the whole layer; the
    // logits are [T, route_E]) and keeps the E of [id_offset, id_offset + E), the rest -1.
    int shard = 0;
    int route_E = 0;
    // optional: counts the one-CTA path zeroes (the FC GEMMs' per-row-block completion counts)
    int32_t *zero_words = nullptr;
    int zero_n = 0;
    __host__ __device__ int routeE() const { return shard ? route_E : E - n_shared; }
};

// Launchers of the forward's kernels.  pdl: launch as programmatic dependents of the kernel
// before them in the stream (each waits for its predecessor before reading its output and lets
// its own successor launch right after that wait); the router, the first kernel of a forward,
// waits for whatever precedes it before it reads the logits or writes the workspace.
// Returns the number of kernels launched (1 for small batches, else 3).
int launch_route_and_group(const RouteGroupArgs &a, cudaStream_t s, bool pdl = false);
// asf_n (optional): the scales again in the N layout of blocks of n_rows rows (sf_n_byte)
void launch_gather(const __nv_bfloat16 *x, int P, int H, int k, const int32_t *pos_of_pair, uint8_t *aq,
                   uint8_t *asf, int act_rows, int act_mxfp8, uint8_t *asf_n, int n_rows, int num_sms,
                   cudaStream_t s, bool pdl = false);
// out: bf16 [T, H], or (out_f32) float32 [T, H]; pairs with pos_of_pair -1 add nothing
void launch_combine(const float *Y, int T, int H, int k, const int32_t *pos_of_pair, const float *topk_w, void *out,
                    int out_f32, int num_sms, cudaStream_t s, bool pdl = false);
void launch_mx_quantize(const float *src, int64_t rows, int64_t K, int fmt, uint8_t *codes, uint8_t *scales,
                        int num_sms, cudaStream_t s);

// Grouped FC GEMM (FC1 with SwiGLU, or FC2) over the row-block list, on
// block-scaled MXFP8 x MXFP4 tensor-core MMAs.
struct FcGemmArgs {
    const int4 *rowblocks;       // {expert, first grouped row, rows, 0}
    const int32_t *num_rowblocks;
    const uint8_t *wscale;       // caller's E8M0 weight scales: [E*R, K/32] row-major, or (wsf_tiled)
                                 // [E][n_tiles][K/128][512] scale atoms (moe_mx_prepare_scales)
    const uint8_t *act_sf;       // activation scale atoms, [rows/128][K/128][2 terms][512]
    uint8_t *hq;                 // FC1 output codes, [2 terms][hq_rows][I] (E4M3)
    uint8_t *hsf;                // FC1 output scale atoms, [hq_rows/128][I/128][2][512]
    float *y;                    // FC2 output, f32 [rows, H]
    uint32_t *err;
    int *unit_counter;           // work-unit counter of this launch, zero before it starts
    unsigned long long timeout_ns;
    int K;                       // reduction length (FC1: H, FC2: I)
    int R;                       // weight rows per expert (FC1: 2I, FC2: H)
    int n_tiles;                 // 128-row weight tiles per expert (FC1: I/64, FC2: H/128)
    int out_ld;                  // leading dimension of the output (FC1: I, FC2: H)
    int act_rows;                // rows of one activation term plane (offset of term 1)
    int hq_rows;                 // rows of one FC1 output term plane
    int terms;                   // activation terms: 2 (w4a16 split) or 1 (w4a8)
    int fc1;                     // 1: gate/up rows + SwiGLU epilogue
    int act_mxfp8;               // FC1 only: h in OCP MXFP8 (w4a8) instead of the two-term split
    int swap_rows;               // row blocks of at most this many rows (<= 128) put the
                                 // weight rows on the MMA M side and the tokens on N
    int wsf_tiled;               // 1: wscale is in the tiled atom layout (one bulk copy per stage)
    int max_block_rows;          // upper bound on any row block's rows: 16, 32, 64 or 128; selects
                                 // the kernel variant (activation tile rows per term)
    int wide;                    // 128-row blocks: two weight tiles per work unit (tokens on M) when
                                 // n_tiles is even
    // FC2 only, every unit with its tokens on N: the weighted combine fused into the epilogue
    // (out = bf16(sum_j w[t,j] * Y[pos(t,j)]) written by the unit that completes a token's k pairs
    // of a weight tile, counted in combine_cnt [T][n_tiles], zero before and after every forward)
    int fuse_combine;
    int *combine_cnt;
    const int32_t *sorted_pair;  // grouped row -> pair t*k + j
    const int32_t *pos_of_pair;  // pair -> grouped row
    const float *topk_w;         // [T, k]
    int k;                       // slots per token
    __nv_bfloat16 *out;          // [T, H]
    // One launch running FC1's units, then FC2's (launch_fc_gemm_two_phase): FC1's epilogue counts
    // each row block's finished units in rb_done (zero before the forward), and an FC2 unit copies
    // its row block's h only once all of them are counted.
    int32_t *rb_done;
    int fc2_tiles;               // FC2 with blocks of <= 16 rows: weight tiles per work unit (2 or 4)
    // Used by the kScalesN kernel instantiations only (launch_fc_gemm picks them when either is
    // set): act_sf_n = the activation scales again in the N layout (sf_n_byte) of blocks of
    // n_rows rows, which units with their tokens on N take with one 512-byte bulk copy per stage
    // instead of 4-byte copies (nullptr: the 4-byte copies); hsf_n = where FC1 also writes h's
    // scales in that layout (nullptr: not written).
    const uint8_t *act_sf_n;
    uint8_t *hsf_n;
    int n_rows;
};

// Tensor maps: act_map = both term planes, 128-row boxes ([terms][128][128] codes, tokens
// on M); act_map_sw = both term planes, boxes of min(max_block_rows, 64) rows (tokens on N);
// act_map16 = 16-row boxes of one plane (tokens on N, blocks beyond that); w_map = FC1: the
// gate and up halves of a 64-row weight slice in one box, FC2: 128-row boxes.
void launch_fc_gemm(const FcGemmArgs &a, const CUtensorMap &act_map, const CUtensorMap &act_map_sw,
                    const CUtensorMap &act_map16, const CUtensorMap &w_map, int grid, cudaStream_t s, bool pdl = false);
cudaError_t fc_gemm_prepare();
// FC1 (a1, with its maps) and FC2 (a2) in one persistent launch, for row blocks of at most 16 rows:
// the work units of FC1 come first, those of FC2 after them, and an FC2 unit waits (bounded) until
// FC1 has finished every unit of its row block.  Both args carry the same rowblocks, rb_done,
// unit counter (one) and error word.
void launch_fc_gemm_two_phase(const FcGemmArgs &a1, const CUtensorMap *maps1, const FcGemmArgs &a2,
                              const CUtensorMap *maps2, int grid, cudaStream_t s, bool pdl);

// Rearrange row-major E8M0 weight scales [E][R][K/32] into the tiled atom layout the GEMM reads:
// for expert e, 128-row weight tile nt and K stage kk (128 elements), one 512-byte atom at
// ((e * n_tiles + nt) * (K/128) + kk) * 512 whose byte sf_atom_offset(m, kb) is the scale of tile
// row m and 32-element block kb.  Tile rows: FC1 (fc1 = 1) gate rows [64 nt, 64 nt + 64) then
// the matching up rows I + [64 nt, 64 nt + 64) (R = 2I); FC2 rows [128 nt, 128 nt + 128).
void launch_tile_scales(const uint8_t *src, uint8_t *dst, int E, int R, int K, int fc1, int num_sms, cudaStream_t s);

void launch_watchdog(uint32_t *err, unsigned long long timeout_ns, cudaStream_t s);

// Encode float32 rows [rows, K] (K a multiple of 128) into codes [2][rows][K] and scale atoms
// [ceil(rows/128)][K/128][2][512] with the forward's activation encoders: method 0 =
// store_act_block32, 1 = store_act_warp32 (test entry moe_mx_debug_encode_act).
void launch_encode_act(const float *src, int rows, int K, int act_mxfp8, int method, uint8_t *q, uint8_t *sf,
                       int num_sms, cudaStream_t s);

// ---------------------------------------------------------------- activation operand format
// Activations reach the tensor core as MXFP8 E4M3 codes in [term][row][K]
// planes plus E8M0 block scales stored in "scale atoms": for every 128 rows x
// 128 K elements, 512 bytes in which tile row m = m0 + 32*m1 (m0 < 32, m1 < 4)
// owns bytes m0*16 + m1*4 + kb (kb = 32-element block within the 128), the
// layout one tcgen05.cp 32x128b.warpx4 moves into TMEM as the MMA expects it.
__device__ __forceinline__ int sf_atom_offset(int m, int kb)
{
    return (m & 31) * 16 + (m >> 5) * 4 + kb;
}

__device__ __forceinline__ size_t sf_atom_byte(int row, int col, int K, int term)
{
    return ((size_t)(row >> 7) * (size_t)(K >> 7) + (size_t)(col >> 7)) * 1024 + (size_t)term * 512 +
           (size_t)sf_atom_offset(row & 127, (col >> 5) & 3);
}

// The N layout, for GEMM units that put a block of n_rows grouped rows (16 or 32, blocks starting
// at multiples of n_rows) on the MMA's N side with both terms side by side: per block and
// 128-element K stage one 512-byte atom, in which row j of term t is the atom's row
// t * n_rows + j.  That is the stage's scale atom as the MMA reads it, so a unit copies it whole.
__device__ __forceinline__ size_t sf_n_byte(int row, int col, int K, int term, int n_rows)
{
    return ((size_t)(row / n_rows) * (size_t)(K >> 7) + (size_t)(col >> 7)) * 512 +
           (size_t)sf_atom_offset(term * n_rows + row % n_rows, (col >> 5) & 3);
}

// E8M0 exponent of a block: floor(log2(amax)) - emax_shift, clamped to [-127, 127]
// (all-zero block: -127).
__device__ __forceinline__ int mx_block_exp(float amax, int emax_shift)
{
    const int s = (amax == 0.f) ? -127 : floor_log2_pos(amax) - emax_shift;
    return max(-127, min(127, s));
}

// Largest finite float: a value compares <= to it only if it is neither infinite nor NaN.
constexpr float kMaxFinite = 3.402823466e38f;

// Encode 32 values as MXFP8 terms.  act_mxfp8 = 1: the OCP rule (shared
// exponent floor(log2 amax) - 8, round-to-nearest-even, saturating) -- one term,
// the w4a8 activation, and the MXFP8 path of moe_mx_quantize.  act_mxfp8 = 0: an
// exact two-term expansion of bf16 values, v = x1 + x2: x1 takes exponent
// floor(log2 amax) - 7 (the block max lands in [128, 256), below the E4M3
// maximum, so nothing saturates) and keeps the top 4 significant bits of every
// element; x2 encodes the remainder v - x1, which has at most 4 significant
// bits, with its own block exponent.  Elements within 2^-13 of the block maximum
// are represented exactly; smaller ones keep an absolute error below 2^-20 of
// the block maximum.  A block that holds a NaN or an infinity has no finite
// scale: every term gets the E8M0 NaN byte 0xFF and zero codes (the OCP
// quantiser's rule for such a block).  The codes come out packed, four to a
// word: element 4i + b in byte b of word i (w0: first term, w1: second).
__device__ __forceinline__ void mx_encode32(const float (&v)[32], int act_mxfp8, uint32_t (&w0)[8], uint32_t (&w1)[8],
                                            uint32_t &s0, uint32_t &s1)
{
    // amax with NaN propagated: the block is finite exactly when amax <= the largest float
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i)
        amax = fmax_nan(amax, fabsf(v[i]));
    if (!(amax <= kMaxFinite)) {
#pragma unroll
        for (int i = 0; i < 8; ++i)
            w0[i] = w1[i] = 0u;
        s0 = s1 = 0xFFu;
        return;
    }
    const int e0 = mx_block_exp(amax, act_mxfp8 ? 8 : 7);
    const float inv0 = exp2_int(-e0), sc0 = exp2_int(e0);
    float r[32];
    float amax1 = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) { // element pairs (2i, 2i + 1): one conversion each way
        const uint32_t p = f32x2_to_e4m3x2(__fmul_rn(v[2 * i], inv0), __fmul_rn(v[2 * i + 1], inv0));
        const float2 d = e4m3x2_to_f32x2(p);
        r[2 * i] = __fsub_rn(v[2 * i], __fmul_rn(d.x, sc0));
        r[2 * i + 1] = __fsub_rn(v[2 * i + 1], __fmul_rn(d.y, sc0));
        amax1 = fmaxf(amax1, fmaxf(fabsf(r[2 * i]), fabsf(r[2 * i + 1])));
        w0[i >> 1] = (i & 1) ? (w0[i >> 1] | (p << 16)) : p;
    }
    s0 = (uint32_t)(e0 + 127);
    if (act_mxfp8) {
#pragma unroll
        for (int i = 0; i < 8; ++i)
            w1[i] = 0u;
        s1 = 0;
        return;
    }
    const int e1 = mx_block_exp(amax1, 7);
    const float inv1 = exp2_int(-e1);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const uint32_t p = f32x2_to_e4m3x2(__fmul_rn(r[2 * i], inv1), __fmul_rn(r[2 * i + 1], inv1));
        w1[i >> 1] = (i & 1) ? (w1[i >> 1] | (p << 16)) : p;
    }
    s1 = (uint32_t)(e1 + 127);
}

__device__ __forceinline__ void store_codes32(uint8_t *dst, const uint32_t (&w)[8])
{
    reinterpret_cast<uint4 *>(dst)[0] = make_uint4(w[0], w[1], w[2], w[3]);
    reinterpret_cast<uint4 *>(dst)[1] = make_uint4(w[4], w[5], w[6], w[7]);
}

// One thread writes the 32-element block [col, col+32) of `row` (values v, f32):
// rounded to bf16 first unless act_mxfp8, then encoded as above.
__device__ __forceinline__ void store_act_block32(uint8_t *q, uint8_t *sf, int plane_rows, int K, int row, int col,
                                                  float (&v)[32], int act_mxfp8)
{
    if (!act_mxfp8) {
#pragma unroll
        for (int i = 0; i < 32; ++i)
            v[i] = __bfloat162float(__float2bfloat16_rn(v[i]));
    }
    uint32_t c0[8], c1[8];
    uint32_t s0, s1;
    mx_encode32(v, act_mxfp8, c0, c1, s0, s1);
    store_codes32(q + (size_t)row * K + col, c0);
    sf[sf_atom_byte(row, col, K, 0)] = (uint8_t)s0;
    if (!act_mxfp8) {
        store_codes32(q + ((size_t)plane_rows + row) * K + col, c1);
        sf[sf_atom_byte(row, col, K, 1)] = (uint8_t)s1;
    }
}

// The 32 lanes of a warp write one 32-element block of `row`, lane l holding
// element col0 + l (col0 = col rounded down to 32): the encoding of
// store_act_block32 computed with warp reductions (same rule, same results).
// sf_n (optional): the scale bytes again in the N layout of blocks of n_rows rows.
__device__ __forceinline__ void store_act_warp32(uint8_t *q, uint8_t *sf, int plane_rows, int K, int row, int col,
                                                 float v, int act_mxfp8, int lane, uint8_t *sf_n = nullptr,
                                                 int n_rows = 0)
{
    if (!act_mxfp8)
        v = __bfloat162float(__float2bfloat16_rn(v));
    const bool finite = __all_sync(0xFFFFFFFFu, fabsf(v) <= kMaxFinite);
    float amax = fabsf(v);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
        amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, off));
    const int e0 = finite ? mx_block_exp(amax, act_mxfp8 ? 8 : 7) : 0;
    const uint32_t c0 = finite ? f32_to_e4m3(__fmul_rn(v, exp2_int(-e0))) : 0u;
    q[(size_t)row * K + col] = (uint8_t)c0;
    if (lane == 0) {
        sf[sf_atom_byte(row, col, K, 0)] = finite ? (uint8_t)(e0 + 127) : (uint8_t)0xFF;
        if (sf_n)
            sf_n[sf_n_byte(row, col, K, 0, n_rows)] = finite ? (uint8_t)(e0 + 127) : (uint8_t)0xFF;
    }
    if (!act_mxfp8) {
        const float r = finite ? __fsub_rn(v, __fmul_rn(e4m3_to_f32(c0), exp2_int(e0))) : 0.f;
        float amax1 = fabsf(r);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
            amax1 = fmaxf(amax1, __shfl_xor_sync(0xFFFFFFFFu, amax1, off));
        const int e1 = mx_block_exp(amax1, 7);
        q[((size_t)plane_rows + row) * K + col] = finite ? (uint8_t)f32_to_e4m3(__fmul_rn(r, exp2_int(-e1))) : 0u;
        if (lane == 0) {
            sf[sf_atom_byte(row, col, K, 1)] = finite ? (uint8_t)(e1 + 127) : (uint8_t)0xFF;
            if (sf_n)
                sf_n[sf_n_byte(row, col, K, 1, n_rows)] = finite ? (uint8_t)(e1 + 127) : (uint8_t)0xFF;
        }
    }
}

} // namespace moe_mx
