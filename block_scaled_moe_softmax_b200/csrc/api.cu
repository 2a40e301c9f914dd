// api.cu -- the C ABI of libmoe_mx.so (declared in include/moe_mx.h): handle
// and workspace management, host-side validation, tensor-map encoding and the
// launch sequence of one forward:
//   route -> scan -> scatter -> gather -> FC1(+SwiGLU) -> FC2 -> combine.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>

#include "../../include/moe_mx.h"
#include "kernels.cuh"

using namespace moe_mx;

namespace {

thread_local std::string g_last_error;

int fail(int code, const char *fmt, ...)
{
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return code;
}

int cuda_fail(cudaError_t e, const char *what)
{
    return fail(MOE_MX_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// 2-D row-major tensor map: inner dimension `cols` elements, `rows` rows,
// `row_bytes` bytes from one row to the next.
// Tensor map of `rank` dimensions (innermost first): dims in elements, strides in bytes of
// dimensions 1..rank-1, box in elements; 128-byte swizzle.
int encode_nd(CUtensorMap *map, CUtensorMapDataType dt, int rank, const void *ptr, const cuuint64_t *dims,
              const cuuint64_t *strides, const cuuint32_t *box)
{
    EncodeTiledFn enc = get_encode_fn();
    if (!enc)
        return fail(MOE_MX_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = enc(map, dt, rank, const_cast<void *>(ptr), dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        return fail(MOE_MX_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d, rank %d)", (int)r, rank);
    return MOE_MX_OK;
}

// 2-D row-major map: `cols` elements per row, `rows` rows, `row_bytes` from one row to the next.
int encode_2d(CUtensorMap *map, CUtensorMapDataType dt, uint64_t row_bytes, const void *ptr, uint64_t cols,
              uint64_t rows, uint32_t box_cols, uint32_t box_rows)
{
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {row_bytes};
    const cuuint32_t box[2] = {box_cols, box_rows};
    return encode_nd(map, dt, 2, ptr, dims, strides, box);
}

// The activation operand as [2 term planes][plane_rows][K] E4M3 codes: boxes of 128 codes x
// box_rows rows x `terms` planes, so one copy brings both terms of a row range.
int encode_act(CUtensorMap *map, const void *ptr, uint64_t K, uint64_t plane_rows, uint32_t box_rows, uint32_t terms)
{
    const cuuint64_t dims[3] = {K, plane_rows, 2};
    const cuuint64_t strides[2] = {K, plane_rows * K};
    const cuuint32_t box[3] = {128, box_rows, terms};
    return encode_nd(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, ptr, dims, strides, box);
}

bool is_device_ptr(const void *p, int dev)
{
    if (!p)
        return false;
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
        cudaGetLastError(); // clear the sticky-free error of an unknown pointer
        return false;
    }
    if (at.type == cudaMemoryTypeManaged)
        return true;
    return at.type == cudaMemoryTypeDevice && at.device == dev;
}

int check_ptr(const void *p, int dev, const char *name)
{
    if (!is_device_ptr(p, dev))
        return fail(MOE_MX_ERR_INVALID_ARG, "%s must be a device pointer on device %d", name, dev);
    if (reinterpret_cast<uintptr_t>(p) % 16 != 0)
        return fail(MOE_MX_ERR_INVALID_ARG, "%s must be 16-byte aligned", name);
    return MOE_MX_OK;
}

int64_t round_up(int64_t v, int64_t m) { return (v + m - 1) / m * m; }

// forwards of at most this many tokens write and read the activation scales in the N layout
constexpr int kScalesNTokens = 16;

int64_t grouped_rows_bound(int E, int64_t pairs)
{
    const int64_t hit = pairs < E ? pairs : E;
    return round_up(pairs + hit * (kBlockRows - 1), kBlockRows);
}

int env_int(const char *name, int dflt)
{
    const char *v = getenv(name);
    return (v && *v) ? atoi(v) : dflt;
}

} // namespace

struct moe_mx_handle {
    // E: expert slots of the weights (routed experts, then the shared expert's S chunks);
    // maxK: the largest routed top-k; a token has top_k + S slots
    int H, I, E, S, maxT, maxK, dev, num_sms;
    int64_t max_rows;
    int64_t n_rows_cap; // grouped rows the N-layout scale buffers cover (forwards of up to kScalesNTokens)
    int swap_rows;
    int tile_rows; // 0: by token count; else 16, 32, 64 or 128 (MOE_MX_TILE_ROWS)
    int pdl;       // launch the kernels after the router as programmatic dependents (MOE_MX_PDL, default 1)
    int wide;      // 128-row GEMM blocks: the two-tile (N = 256) variant (MOE_MX_WIDE, default 1)
    int fuse_combine; // small batches: the combine in FC2's epilogue (MOE_MX_FUSE_COMBINE; off by default: slower)
    int two_phase;    // small batches: FC1 and FC2 in one launch (MOE_MX_TWO_PHASE, default 1)
    int two_phase_max_tokens; // ... up to this many tokens (at most 16)
    int scales_n;             // N-layout activation scales up to 16 tokens (MOE_MX_SCALES_N, default 1)
    int fc2_tiles;            // FC2 of blocks of <= 16 rows: weight tiles per unit (MOE_MX_FC2_TILES: 0 = by
                              // token count, 2 or 4)
    int scale_layout; // MOE_MX_SCALES_ROW_MAJOR or MOE_MX_SCALES_TILED
    unsigned long long timeout_ns;
    void *ws;
    int32_t *topk_ids, *chunk_hist, *counts, *pad_offsets, *num_rowblocks, *sorted_pair, *pos_of_pair;
    int32_t *unit_counters;
    int32_t *combine_cnt; // [max_tokens][H/128] pairs of each token and FC2 weight tile done (fused combine)
    int32_t *rb_done;     // [max_rows/16] FC1 units done per row block (two-phase launch)
    float *topk_w;
    int4 *rowblocks;
    uint8_t *Aq, *Asf, *Hq, *Hsf; // MXFP8 operand planes [2][rows][K] and their scale atoms
    uint8_t *AsfN, *HsfN;         // the same scales in the N layout (forwards with 16- or 32-row blocks)
    float *Y;
    uint32_t *err;
    // activation operands: [terms - 1] 128-row boxes; [terms - 1][kT2 16/32/64] boxes for tokens
    // on N; 16-row single-plane boxes
    CUtensorMap map_A[2], map_Asw[2][3], map_A16, map_H[2], map_Hsw[2][3], map_H16;
    const void *w1_key, *w2_key;
    CUtensorMap map_w1, map_w2;
    int last_T, last_k;
    long long launches; // kernels launched by this handle's forwards since create
    // stage timing: a ring of kTimingRing event sets, one set per timed forward
    cudaEvent_t *ev;
    bool timing;
    long long n_timed;
};

namespace {
constexpr int kTimingRing = 1024;
constexpr int kEvPerFwd = MOE_MX_NUM_STAGES + 1;
} // namespace

extern "C" {

const char *moe_mx_last_error(void) { return g_last_error.c_str(); }

int moe_mx_block_rows(void) { return kBlockRows; }

int64_t moe_mx_max_grouped_rows(const moe_mx_handle *h, int num_tokens, int top_k)
{
    if (!h || num_tokens < 0 || top_k < 1)
        return 0;
    return grouped_rows_bound(h->E, (int64_t)num_tokens * (top_k + h->S));
}

int moe_mx_create(moe_mx_handle **out, int hidden, int inter, int num_experts, int max_tokens, int max_top_k,
                  int device)
{
    return moe_mx_create_ex(out, hidden, inter, num_experts, 0, max_tokens, max_top_k, device);
}

int moe_mx_create_ex(moe_mx_handle **out, int hidden, int inter, int num_experts, int num_shared, int max_tokens,
                     int max_top_k, int device)
{
    g_last_error.clear();
    if (!out)
        return fail(MOE_MX_ERR_INVALID_ARG, "out is NULL");
    *out = nullptr;
    if (hidden < 128 || hidden > 16384 || hidden % 128 != 0)
        return fail(MOE_MX_ERR_UNSUPPORTED, "hidden=%d must be a multiple of 128 in [128, 16384]", hidden);
    if (inter < 128 || inter > 8192 || inter % 128 != 0)
        return fail(MOE_MX_ERR_UNSUPPORTED, "inter=%d must be a multiple of 128 in [128, 8192]", inter);
    if (num_experts < 1 || num_experts > kMaxExperts)
        return fail(MOE_MX_ERR_UNSUPPORTED, "num_experts=%d must be in [1, %d]", num_experts, kMaxExperts);
    if (max_tokens < 1 || max_tokens > 65536)
        return fail(MOE_MX_ERR_INVALID_ARG, "max_tokens=%d must be in [1, 65536]", max_tokens);
    if (max_top_k < 1 || max_top_k > kMaxTopK)
        return fail(MOE_MX_ERR_INVALID_ARG, "max_top_k=%d must be in [1, %d]", max_top_k, kMaxTopK);
    if (num_shared < 0 || num_experts + num_shared > kMaxExperts || max_top_k + num_shared > kMaxTopK)
        return fail(MOE_MX_ERR_UNSUPPORTED,
                    "num_shared=%d: need num_experts + num_shared <= %d and max_top_k + num_shared <= %d",
                    num_shared, kMaxExperts, kMaxTopK);
    int ndev = 0;
    cudaError_t ce = cudaGetDeviceCount(&ndev);
    if (ce != cudaSuccess)
        return cuda_fail(ce, "cudaGetDeviceCount");
    if (device < 0 || device >= ndev)
        return fail(MOE_MX_ERR_INVALID_ARG, "device %d out of range (%d devices)", device, ndev);
    cudaDeviceProp prop;
    if ((ce = cudaGetDeviceProperties(&prop, device)) != cudaSuccess)
        return cuda_fail(ce, "cudaGetDeviceProperties");
    if (prop.major != 10 || prop.minor != 0)
        return fail(MOE_MX_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library is built for sm_100a", device,
                    prop.major, prop.minor);
    int prev = 0;
    cudaGetDevice(&prev);
    if ((ce = cudaSetDevice(device)) != cudaSuccess)
        return cuda_fail(ce, "cudaSetDevice");

    moe_mx_handle *h = new moe_mx_handle();
    h->H = hidden;
    h->I = inter;
    h->E = num_experts + num_shared;
    h->S = num_shared;
    h->maxT = max_tokens;
    h->maxK = max_top_k;
    h->dev = device;
    h->num_sms = prop.multiProcessorCount;
    const int64_t pairs = (int64_t)max_tokens * (max_top_k + num_shared);
    h->max_rows = grouped_rows_bound(h->E, pairs);
    h->n_rows_cap = grouped_rows_bound(
        h->E, (int64_t)(max_tokens < kScalesNTokens ? max_tokens : kScalesNTokens) * (max_top_k + num_shared));
    h->scale_layout = MOE_MX_SCALES_ROW_MAJOR;
    h->tile_rows = env_int("MOE_MX_TILE_ROWS", 0);
    if (h->tile_rows != 16 && h->tile_rows != 32 && h->tile_rows != 64 && h->tile_rows != kBlockRows)
        h->tile_rows = 0;
    h->pdl = env_int("MOE_MX_PDL", 1) != 0;
    h->wide = env_int("MOE_MX_WIDE", 1) != 0;
    h->fuse_combine = env_int("MOE_MX_FUSE_COMBINE", 0) != 0;
    h->two_phase = env_int("MOE_MX_TWO_PHASE", 1) != 0;
    // measured: one launch gains at 1 and 2 tokens (1 token 0.090 -> 0.083 ms; 2 tokens, with the
    // N-layout scales, 0.1228 -> 0.1195 ms) and loses from 4 tokens on (0.172 -> 0.188 ms: its FC2
    // units are one weight tile each, and short); MOE_MX_TWO_PHASE_TOKENS (<= 16) moves the bound
    h->two_phase_max_tokens = env_int("MOE_MX_TWO_PHASE_TOKENS", 2);
    h->scales_n = env_int("MOE_MX_SCALES_N", 1) != 0;
    h->fc2_tiles = env_int("MOE_MX_FC2_TILES", 0);
    if (h->fc2_tiles != 2 && h->fc2_tiles != 4)
        h->fc2_tiles = 0;
    if (h->two_phase_max_tokens > 16)
        h->two_phase_max_tokens = 16;
    h->swap_rows = env_int("MOE_MX_SWAP_ROWS", 64);
    if (h->swap_rows < 0)
        h->swap_rows = 0;
    if (h->swap_rows > kBlockRows)
        h->swap_rows = kBlockRows;
    h->timeout_ns = (unsigned long long)env_int("MOE_MX_TIMEOUT_MS", 2000) * 1000000ull;

    const int64_t nchunks = (max_tokens + kRouteChunk - 1) / kRouteChunk;
    struct Part {
        void **dst;
        size_t bytes;
    } parts[] = {
        {(void **)&h->topk_ids, sizeof(int32_t) * pairs},
        {(void **)&h->topk_w, sizeof(float) * pairs},
        {(void **)&h->chunk_hist, sizeof(int32_t) * nchunks * h->E},
        {(void **)&h->counts, sizeof(int32_t) * h->E},
        {(void **)&h->pad_offsets, sizeof(int32_t) * (h->E + 1)},
        {(void **)&h->rowblocks, sizeof(int4) * (h->max_rows / 16)}, // work blocks: >= 16 padded rows each
        {(void **)&h->num_rowblocks, sizeof(int32_t)},
        {(void **)&h->unit_counters, 2 * sizeof(int32_t)}, // FC1, FC2 work-unit counters
        {(void **)&h->combine_cnt, sizeof(int32_t) * max_tokens * (hidden / 128)},
        {(void **)&h->rb_done, sizeof(int32_t) * (h->max_rows / 16)},
        {(void **)&h->sorted_pair, sizeof(int32_t) * h->max_rows},
        {(void **)&h->pos_of_pair, sizeof(int32_t) * pairs},
        {(void **)&h->err, sizeof(uint32_t)},
        {(void **)&h->Aq, (size_t)2 * h->max_rows * hidden},
        {(void **)&h->Asf, (size_t)(h->max_rows / 128) * (hidden / 128) * 1024},
        {(void **)&h->Hq, (size_t)2 * h->max_rows * inter},
        {(void **)&h->Hsf, (size_t)(h->max_rows / 128) * (inter / 128) * 1024},
        {(void **)&h->Y, sizeof(float) * h->max_rows * hidden},
        // x's and h's scales again in the N layout of 16-row blocks (32-row blocks take half)
        {(void **)&h->AsfN, (size_t)(h->n_rows_cap / 16) * (hidden / 128) * 512},
        {(void **)&h->HsfN, (size_t)(h->n_rows_cap / 16) * (inter / 128) * 512},
    };
    size_t total = 0;
    for (auto &p : parts)
        total += round_up((int64_t)p.bytes, 1024);
    if ((ce = cudaMalloc(&h->ws, total)) != cudaSuccess) {
        cudaGetLastError();
        delete h;
        cudaSetDevice(prev);
        return fail(MOE_MX_ERR_NO_MEMORY, "cudaMalloc of %zu workspace bytes failed", total);
    }
    size_t off = 0;
    for (auto &p : parts) {
        *p.dst = static_cast<uint8_t *>(h->ws) + off;
        off += round_up((int64_t)p.bytes, 1024);
    }
    int rc = MOE_MX_OK;
    if ((ce = cudaMemset(h->ws, 0, total)) != cudaSuccess)
        rc = cuda_fail(ce, "cudaMemset(workspace)");
    if (rc == MOE_MX_OK && (ce = fc_gemm_prepare()) != cudaSuccess)
        rc = cuda_fail(ce, "cudaFuncSetAttribute(fc_gemm)");
    // activation operand planes: [2 terms x rows, K] E4M3 codes (128-byte swizzle = the K-major
    // layout the MMA reads): boxes over both planes of 128 rows (tokens on M) or of 16, 32 or 64
    // rows (tokens on N), and 16-row single-plane boxes
    for (int t = 1; t <= 2 && rc == MOE_MX_OK; ++t) {
        rc = encode_act(&h->map_A[t - 1], h->Aq, hidden, h->max_rows, 128, t);
        for (int i = 0; i < 3 && rc == MOE_MX_OK; ++i)
            rc = encode_act(&h->map_Asw[t - 1][i], h->Aq, hidden, h->max_rows, 16u << i, t);
    }
    for (int t = 1; t <= 2 && rc == MOE_MX_OK; ++t) {
        rc = encode_act(&h->map_H[t - 1], h->Hq, inter, h->max_rows, 128, t);
        for (int i = 0; i < 3 && rc == MOE_MX_OK; ++i)
            rc = encode_act(&h->map_Hsw[t - 1][i], h->Hq, inter, h->max_rows, 16u << i, t);
    }
    if (rc == MOE_MX_OK)
        rc = encode_2d(&h->map_A16, CU_TENSOR_MAP_DATA_TYPE_UINT8, hidden, h->Aq, hidden, 2 * h->max_rows, 128, 16);
    if (rc == MOE_MX_OK)
        rc = encode_2d(&h->map_H16, CU_TENSOR_MAP_DATA_TYPE_UINT8, inter, h->Hq, inter, 2 * h->max_rows, 128, 16);
    if (rc == MOE_MX_OK && (ce = cudaDeviceSynchronize()) != cudaSuccess)
        rc = cuda_fail(ce, "cudaDeviceSynchronize(create)");
    cudaSetDevice(prev);
    if (rc != MOE_MX_OK) {
        cudaFree(h->ws);
        delete h;
        return rc;
    }
    *out = h;
    return MOE_MX_OK;
}

int moe_mx_destroy(moe_mx_handle *h)
{
    if (!h)
        return MOE_MX_OK;
    int prev = 0;
    cudaGetDevice(&prev);
    cudaSetDevice(h->dev);
    cudaDeviceSynchronize();
    if (h->timing) {
        for (int i = 0; i < kTimingRing * kEvPerFwd; ++i)
            cudaEventDestroy(h->ev[i]);
        delete[] h->ev;
    }
    cudaFree(h->ws);
    cudaSetDevice(prev);
    delete h;
    return MOE_MX_OK;
}

namespace {

// The forward of every entry point: routing computed from router_logits, or (given_ids set)
// the given global ids and weights restricted to the shard [id_offset, id_offset + E); with
// route_E > 0 the logits cover route_E experts (the whole layer) and the routed pairs are
// restricted to the shard [id_offset, id_offset + E) the handle holds.
int forward_impl(moe_mx_handle *h, const void *x, const float *router_logits, const int32_t *given_ids,
                 const float *given_w, int id_offset, int num_tokens, const uint8_t *w1, const uint8_t *w1_scale,
                 const uint8_t *w2, const uint8_t *w2_scale, int top_k, int act_dtype, void *out, int out_f32,
                 void *stream, int route_E = 0)
{
    g_last_error.clear();
    if (!h)
        return fail(MOE_MX_ERR_INVALID_ARG, "handle is NULL");
    if (num_tokens < 0 || num_tokens > h->maxT)
        return fail(MOE_MX_ERR_INVALID_ARG, "num_tokens=%d must be in [0, %d]", num_tokens, h->maxT);
    if (route_E > 0 && h->S > 0)
        return fail(MOE_MX_ERR_UNSUPPORTED, "the shard form takes no shared expert (handle has %d shared chunks)",
                    h->S);
    if (route_E > 0 && (route_E > kMaxExperts || id_offset < 0 || id_offset > route_E - h->E))
        return fail(MOE_MX_ERR_INVALID_ARG,
                    "num_experts_global=%d, local_expert_offset=%d: need the shard [offset, offset + %d) inside "
                    "[0, num_experts_global) and num_experts_global <= %d",
                    route_E, id_offset, h->E, kMaxExperts);
    const int routed = route_E > 0 ? route_E : h->E - h->S; // experts the router chooses among
    if (!given_ids && (top_k < 1 || top_k > h->maxK || top_k > routed))
        return fail(MOE_MX_ERR_INVALID_ARG, "top_k=%d must be in [1, min(E=%d, max_top_k=%d)]", top_k, routed,
                    h->maxK);
    if (given_ids && h->S > 0)
        return fail(MOE_MX_ERR_UNSUPPORTED, "the routed form takes no shared expert (handle has %d shared chunks)",
                    h->S);
    if (given_ids && (top_k < 1 || top_k > h->maxK))
        return fail(MOE_MX_ERR_INVALID_ARG, "top_k=%d must be in [1, max_top_k=%d]", top_k, h->maxK);
    if (given_ids && id_offset < 0)
        return fail(MOE_MX_ERR_INVALID_ARG, "local_expert_offset=%d must be >= 0", id_offset);
    if (act_dtype != MOE_MX_ACT_BF16 && act_dtype != MOE_MX_ACT_MXFP8)
        return fail(MOE_MX_ERR_INVALID_ARG, "act_dtype=%d is not MOE_MX_ACT_BF16 or MOE_MX_ACT_MXFP8", act_dtype);
    if (num_tokens == 0)
        return MOE_MX_OK;
    int rc;
    if (given_ids) {
        if ((rc = check_ptr(given_ids, h->dev, "topk_ids")) || (rc = check_ptr(given_w, h->dev, "topk_w")))
            return rc;
    } else if ((rc = check_ptr(router_logits, h->dev, "router_logits"))) {
        return rc;
    }
    if ((rc = check_ptr(x, h->dev, "x")) ||
        (rc = check_ptr(w1, h->dev, "w1")) || (rc = check_ptr(w1_scale, h->dev, "w1_scale")) ||
        (rc = check_ptr(w2, h->dev, "w2")) || (rc = check_ptr(w2_scale, h->dev, "w2_scale")) ||
        (rc = check_ptr(out, h->dev, "out")))
        return rc;
    if (x == out)
        return fail(MOE_MX_ERR_INVALID_ARG, "out must not alias x");
    if (reinterpret_cast<uintptr_t>(w1) % 32 != 0 || reinterpret_cast<uintptr_t>(w2) % 32 != 0)
        return fail(MOE_MX_ERR_INVALID_ARG, "w1 and w2 must be 32-byte aligned");

    // E: expert slots; k: slots per token (the routed top_k, then the shared expert's chunks)
    const int H = h->H, I = h->I, E = h->E, T = num_tokens, k = top_k + h->S;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int prev = 0;
    cudaGetDevice(&prev);
    if (prev != h->dev)
        cudaSetDevice(h->dev);

    // weights: packed E2M1 [rows, K] unpacked by the TMA into 8-bit containers (16 codes per
    // 16-byte granule), 128-byte swizzle.  W1 as [2E halves][I rows][H] so that one box of
    // 128 codes x 64 rows x 2 halves brings a gate slice and its up slice; W2 in 128-row boxes.
    if (w1 != h->w1_key) {
        const cuuint64_t dims[3] = {(cuuint64_t)H, (cuuint64_t)I, (cuuint64_t)2 * E};
        const cuuint64_t strides[2] = {(cuuint64_t)H / 2, (cuuint64_t)I * (H / 2)};
        const cuuint32_t box[3] = {128, 64, 2};
        if ((rc = encode_nd(&h->map_w1, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 3, w1, dims, strides, box)))
            goto done;
        h->w1_key = w1;
    }
    if (w2 != h->w2_key) {
        if ((rc = encode_2d(&h->map_w2, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, I / 2, w2, I, (uint64_t)E * H, 128,
                            128)))
            goto done;
        h->w2_key = w2;
    }
    {
        const int64_t pairs = (int64_t)T * k;
        cudaError_t ce;
        cudaEvent_t *evset = h->timing ? h->ev + (h->n_timed % kTimingRing) * kEvPerFwd : nullptr;
        auto mark = [&](int i) {
            if (evset)
                cudaEventRecord(evset[i], s);
        };
        mark(0);
        // activation tile rows per term of the GEMM variant; the segments are split into work
        // blocks of at most that many rows (a segment holds one expert's tokens, so at 16 tokens
        // nothing is split).  Up to a few hundred tokens small blocks, all with their tokens on N,
        // are fastest: re-reading the weights of the few experts split into several blocks costs
        // less than the deeper pipelines gain.  Measured at 256 tokens: 32-row blocks 1.61 ms
        // against 1.90 ms with 64-row ones, and 16-row blocks (FC2 then takes four weight tiles
        // per unit) 1.48 ms against 1.56 ms with 32-row ones.
        const int tile_rows = h->tile_rows > 0 ? h->tile_rows
                              : T <= 256       ? 16
                              : T <= 512       ? 32
                                               : kBlockRows;
        RouteGroupArgs ra{router_logits, T, E, k, h->topk_ids, h->topk_w, h->chunk_hist, h->counts,
                          h->pad_offsets, h->rowblocks, h->num_rowblocks, h->sorted_pair, h->pos_of_pair,
                          tile_rows, h->unit_counters};
        ra.given_ids = given_ids;
        ra.given_w = given_w;
        ra.id_offset = id_offset;
        ra.n_shared = h->S;
        ra.shard = route_E > 0;
        ra.route_E = route_E;
        // Up to 16 tokens routed from logits (the k experts of a token distinct), every expert's
        // pairs fit one 16-row block: FC1 and FC2 then run as one launch (two phases), FC2's units
        // waiting for their row block's FC1 units through rb_done, which the routing kernel (one
        // CTA at this size) zeroes.  Row blocks: at most one per expert slot hit.
        const bool two = h->two_phase && !given_ids && tile_rows == 16 && T <= h->two_phase_max_tokens;
        if (two) {
            ra.zero_words = h->rb_done;
            ra.zero_n = (int)((int64_t)T * k < E ? (int64_t)T * k : E);
        }
        // Each kernel may launch while its predecessor still runs (programmatic dependent launch):
        // the FC GEMMs start streaming their weights early, and the router's launch overlaps the
        // tail of whatever precedes the forward in the stream (it waits for it before its work).
        // Stage timing records events between the kernels, so timed forwards launch them one after
        // another.
        const bool pdl = h->pdl && !evset;
        h->launches += launch_route_and_group(ra, s, pdl);
        mark(1);
        const int mx8 = act_dtype == MOE_MX_ACT_MXFP8;
        // Up to 16 tokens (16-row blocks, tokens on N) the gather and FC1 also write the activation
        // scales in the N layout, so that a GEMM stage takes them with one bulk copy instead of
        // 4-byte copies.  Measured: 1 token 0.0826 -> 0.0757 ms, 4 tokens 0.1739 ->
        // 0.1712, 16 tokens 0.4522 -> 0.4515; at 256 tokens slower (1.455 -> 1.48 ms), so the
        // 4-byte copies stay there.
        const bool scales_n = h->scales_n && tile_rows == 16 && T <= kScalesNTokens &&
                              grouped_rows_bound(E, pairs) <= h->n_rows_cap;
        launch_gather(static_cast<const __nv_bfloat16 *>(x), (int)pairs, H, k, h->pos_of_pair, h->Aq, h->Asf,
                      (int)h->max_rows, mx8, scales_n ? h->AsfN : nullptr, tile_rows, h->num_sms, s, pdl);

        FcGemmArgs f1{};
        f1.rowblocks = h->rowblocks;
        f1.num_rowblocks = h->num_rowblocks;
        f1.wscale = w1_scale;
        f1.wsf_tiled = h->scale_layout == MOE_MX_SCALES_TILED;
        f1.unit_counter = h->unit_counters;
        f1.act_sf = h->Asf;
        f1.hq = h->Hq;
        f1.hsf = h->Hsf;
        f1.y = h->Y;
        f1.err = h->err;
        f1.timeout_ns = h->timeout_ns;
        f1.K = H;
        f1.R = 2 * I;
        f1.n_tiles = I / 64;
        f1.out_ld = I;
        f1.act_rows = (int)h->max_rows;
        f1.hq_rows = (int)h->max_rows;
        f1.terms = mx8 ? 1 : 2;
        f1.fc1 = 1;
        f1.act_mxfp8 = mx8;
        f1.swap_rows = h->swap_rows;
        f1.max_block_rows = tile_rows;
        f1.wide = h->wide;
        f1.act_sf_n = scales_n ? h->AsfN : nullptr;
        f1.hsf_n = scales_n ? h->HsfN : nullptr;
        f1.n_rows = tile_rows;
        mark(2);
        const int sw_idx = tile_rows <= 16 ? 0 : tile_rows <= 32 ? 1 : 2; // box rows min(tile rows, 64)
        if (!two)
            launch_fc_gemm(f1, h->map_A[f1.terms - 1], h->map_Asw[f1.terms - 1][sw_idx], h->map_A16, h->map_w1,
                           h->num_sms, s, pdl);
        if (!two)
            mark(3);

        FcGemmArgs f2 = f1;
        f2.act_sf_n = scales_n ? h->HsfN : nullptr;
        f2.hsf_n = nullptr;
        f2.wscale = w2_scale;
        f2.unit_counter = h->unit_counters + 1;
        f2.act_sf = h->Hsf;
        f2.K = I;
        f2.R = H;
        f2.n_tiles = H / 128;
        f2.out_ld = H;
        f2.fc1 = 0;
        f2.act_mxfp8 = 0;
        // FC2 of 16-row blocks: four weight tiles per unit (3 stages of 4 tiles: 96 KB of weights in
        // flight per SM, against 80 KB in 5 stages of 2) when there are many units to share out;
        // measured at 16 tokens 164 -> 145 us, at 2 and 4 tokens no gain
        f2.fc2_tiles = h->fc2_tiles ? h->fc2_tiles : (T > 4 ? 4 : 2);
        // small batches of the logits form: every FC2 unit has its tokens on N, and its epilogue
        // finishes the combine of the tokens whose k pairs it completes
        const bool fuse = h->fuse_combine && !given_ids && route_E == 0 && tile_rows <= 64;
        f2.fuse_combine = fuse;
        f2.combine_cnt = h->combine_cnt;
        f2.sorted_pair = h->sorted_pair;
        f2.pos_of_pair = h->pos_of_pair;
        f2.topk_w = h->topk_w;
        f2.k = k;
        f2.out = static_cast<__nv_bfloat16 *>(out);
        // the maps' plane count must equal the copy's terms: the stage barrier expects exactly those bytes
        if (two) {
            // one launch, one work-unit counter: FC1's units first, then FC2's
            f1.rb_done = f2.rb_done = h->rb_done;
            f2.unit_counter = f1.unit_counter;
            const CUtensorMap m1[4] = {h->map_A[f1.terms - 1], h->map_Asw[f1.terms - 1][sw_idx], h->map_A16,
                                       h->map_w1};
            const CUtensorMap m2[4] = {h->map_H[f2.terms - 1], h->map_Hsw[f2.terms - 1][sw_idx], h->map_H16,
                                       h->map_w2};
            launch_fc_gemm_two_phase(f1, m1, f2, m2, h->num_sms, s, pdl);
            mark(3); // the FC1 stage's time covers both GEMMs; the FC2 stage is empty
        } else {
            launch_fc_gemm(f2, h->map_H[f2.terms - 1], h->map_Hsw[f2.terms - 1][sw_idx], h->map_H16, h->map_w2,
                           h->num_sms, s, pdl);
        }
        mark(4);
        if (!fuse)
            launch_combine(h->Y, T, H, k, h->pos_of_pair, h->topk_w, out, out_f32, h->num_sms, s, pdl);
        h->launches += 1 + (two ? 1 : 2) + (fuse ? 0 : 1); // gather, FC1 and FC2 (one launch or two), combine
        ce = cudaGetLastError();
        if (ce != cudaSuccess) {
            rc = cuda_fail(ce, "kernel launch");
            goto done;
        }
        mark(5);
        h->last_T = T;
        h->last_k = k;
        if (h->timing)
            ++h->n_timed;
    }
done:
    if (prev != h->dev)
        cudaSetDevice(prev);
    return rc;
}

} // namespace

int moe_mx_forward(moe_mx_handle *h, const void *x, const float *router_logits, int num_tokens, const uint8_t *w1,
                   const uint8_t *w1_scale, const uint8_t *w2, const uint8_t *w2_scale, int top_k, int act_dtype,
                   void *out, void *stream)
{
    return forward_impl(h, x, router_logits, nullptr, nullptr, 0, num_tokens, w1, w1_scale, w2, w2_scale, top_k,
                        act_dtype, out, 0, stream);
}

int moe_mx_forward_routed(moe_mx_handle *h, const void *x, const int32_t *topk_ids, const float *topk_w,
                          int num_tokens, int top_k, int local_expert_offset, const uint8_t *w1,
                          const uint8_t *w1_scale, const uint8_t *w2, const uint8_t *w2_scale, int act_dtype,
                          void *out, int out_dtype, void *stream)
{
    if (out_dtype != MOE_MX_OUT_BF16 && out_dtype != MOE_MX_OUT_F32) {
        g_last_error.clear();
        return fail(MOE_MX_ERR_INVALID_ARG, "out_dtype=%d is not MOE_MX_OUT_BF16 or MOE_MX_OUT_F32", out_dtype);
    }
    if (!topk_ids || !topk_w) {
        g_last_error.clear();
        return fail(MOE_MX_ERR_INVALID_ARG, "topk_ids and topk_w must not be NULL");
    }
    return forward_impl(h, x, nullptr, topk_ids, topk_w, local_expert_offset, num_tokens, w1, w1_scale, w2, w2_scale,
                        top_k, act_dtype, out, out_dtype == MOE_MX_OUT_F32, stream);
}

int moe_mx_forward_shard(moe_mx_handle *h, const void *x, const float *router_logits, int num_tokens,
                         int num_experts_global, int local_expert_offset, const uint8_t *w1, const uint8_t *w1_scale,
                         const uint8_t *w2, const uint8_t *w2_scale, int top_k, int act_dtype, void *out,
                         int out_dtype, void *stream)
{
    if (out_dtype != MOE_MX_OUT_BF16 && out_dtype != MOE_MX_OUT_F32) {
        g_last_error.clear();
        return fail(MOE_MX_ERR_INVALID_ARG, "out_dtype=%d is not MOE_MX_OUT_BF16 or MOE_MX_OUT_F32", out_dtype);
    }
    if (num_experts_global < 1) {
        g_last_error.clear();
        return fail(MOE_MX_ERR_INVALID_ARG, "num_experts_global=%d must be >= 1", num_experts_global);
    }
    return forward_impl(h, x, router_logits, nullptr, nullptr, local_expert_offset, num_tokens, w1, w1_scale, w2,
                        w2_scale, top_k, act_dtype, out, out_dtype == MOE_MX_OUT_F32, stream, num_experts_global);
}

int moe_mx_sync_status(moe_mx_handle *h, void *stream)
{
    g_last_error.clear();
    if (!h)
        return fail(MOE_MX_ERR_INVALID_ARG, "handle is NULL");
    cudaError_t ce = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (ce != cudaSuccess)
        return cuda_fail(ce, "cudaStreamSynchronize");
    uint32_t word = 0;
    if ((ce = cudaMemcpy(&word, h->err, sizeof(word), cudaMemcpyDeviceToHost)) != cudaSuccess)
        return cuda_fail(ce, "cudaMemcpy(error word)");
    if (word != 0) {
        // a forward cut short may leave the fused combine's counts behind: they start at zero again
        cudaMemset(h->combine_cnt, 0, sizeof(int32_t) * h->maxT * (h->H / 128));
        cudaMemset(h->err, 0, sizeof(uint32_t));
        cudaDeviceSynchronize();
        return fail(MOE_MX_ERR_TIMEOUT, "a device-side wait gave up (error word 0x%x)", word);
    }
    return MOE_MX_OK;
}

int moe_mx_quantize(const float *src, int64_t rows, int64_t K, int fmt, uint8_t *codes, uint8_t *scales,
                    void *stream)
{
    g_last_error.clear();
    if (rows < 0 || K <= 0 || K % 32 != 0)
        return fail(MOE_MX_ERR_INVALID_ARG, "rows=%lld K=%lld: K must be a positive multiple of 32",
                    (long long)rows, (long long)K);
    if (fmt != MOE_MX_FMT_MXFP4 && fmt != MOE_MX_FMT_MXFP8)
        return fail(MOE_MX_ERR_INVALID_ARG, "fmt=%d is not MOE_MX_FMT_MXFP4 or MOE_MX_FMT_MXFP8", fmt);
    if (rows == 0)
        return MOE_MX_OK;
    int dev = 0;
    cudaGetDevice(&dev);
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, src) == cudaSuccess && at.type == cudaMemoryTypeDevice)
        dev = at.device;
    else
        cudaGetLastError();
    int rc;
    if ((rc = check_ptr(src, dev, "src")) || (rc = check_ptr(codes, dev, "codes")) ||
        (rc = check_ptr(scales, dev, "scales")))
        return rc;
    int nsm = 148;
    cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    int prev = 0;
    cudaGetDevice(&prev);
    if (prev != dev)
        cudaSetDevice(dev);
    launch_mx_quantize(src, rows, K, fmt, codes, scales, nsm, static_cast<cudaStream_t>(stream));
    cudaError_t ce = cudaGetLastError();
    if (prev != dev)
        cudaSetDevice(prev);
    if (ce != cudaSuccess)
        return cuda_fail(ce, "mx_quantize launch");
    return MOE_MX_OK;
}

int moe_mx_get_routing(const moe_mx_handle *h, int32_t *topk_ids, float *topk_w, int32_t *counts,
                       int32_t *pad_offsets, int32_t *sorted_pair, void *stream)
{
    g_last_error.clear();
    if (!h)
        return fail(MOE_MX_ERR_INVALID_ARG, "handle is NULL");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int64_t pairs = (int64_t)h->last_T * h->last_k;
    struct Copy {
        void *dst;
        const void *src;
        size_t bytes;
        const char *name;
    } copies[] = {
        {topk_ids, h->topk_ids, sizeof(int32_t) * pairs, "topk_ids"},
        {topk_w, h->topk_w, sizeof(float) * pairs, "topk_w"},
        {counts, h->counts, sizeof(int32_t) * h->E, "counts"},
        {pad_offsets, h->pad_offsets, sizeof(int32_t) * (h->E + 1), "pad_offsets"},
        {sorted_pair, h->sorted_pair, sizeof(int32_t) * grouped_rows_bound(h->E, pairs), "sorted_pair"},
    };
    for (auto &c : copies) {
        if (!c.dst || c.bytes == 0)
            continue;
        if (!is_device_ptr(c.dst, h->dev))
            return fail(MOE_MX_ERR_INVALID_ARG, "%s must be a device pointer on device %d", c.name, h->dev);
        cudaError_t ce = cudaMemcpyAsync(c.dst, c.src, c.bytes, cudaMemcpyDeviceToDevice, s);
        if (ce != cudaSuccess)
            return cuda_fail(ce, "cudaMemcpyAsync(routing state)");
    }
    return MOE_MX_OK;
}

int moe_mx_get_intermediate(const moe_mx_handle *h, int which, void *dst, void *stream)
{
    g_last_error.clear();
    if (!h)
        return fail(MOE_MX_ERR_INVALID_ARG, "handle is NULL");
    if (which < MOE_MX_INTER_AQ || which > MOE_MX_INTER_Y)
        return fail(MOE_MX_ERR_INVALID_ARG, "which=%d is not one of MOE_MX_INTER_*", which);
    const int64_t rows = grouped_rows_bound(h->E, (int64_t)h->last_T * h->last_k);
    if (rows == 0)
        return MOE_MX_OK;
    if (!is_device_ptr(dst, h->dev))
        return fail(MOE_MX_ERR_INVALID_ARG, "dst must be a device pointer on device %d", h->dev);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int64_t K = (which == MOE_MX_INTER_AQ || which == MOE_MX_INTER_ASF) ? h->H : h->I;
    cudaError_t ce = cudaSuccess;
    uint8_t *d = static_cast<uint8_t *>(dst);
    if (which == MOE_MX_INTER_AQ || which == MOE_MX_INTER_HQ) {
        // two term planes of `rows` rows each, packed; in the workspace they sit max_rows apart
        const uint8_t *src = which == MOE_MX_INTER_AQ ? h->Aq : h->Hq;
        for (int t = 0; t < 2 && ce == cudaSuccess; ++t)
            ce = cudaMemcpyAsync(d + t * rows * K, src + t * h->max_rows * K, (size_t)(rows * K),
                                 cudaMemcpyDeviceToDevice, s);
    } else if (which == MOE_MX_INTER_ASF || which == MOE_MX_INTER_HSF) {
        const uint8_t *src = which == MOE_MX_INTER_ASF ? h->Asf : h->Hsf;
        ce = cudaMemcpyAsync(d, src, (size_t)((rows / 128) * (K / 128) * 1024), cudaMemcpyDeviceToDevice, s);
    } else {
        ce = cudaMemcpyAsync(d, h->Y, (size_t)(rows * h->H) * sizeof(float), cudaMemcpyDeviceToDevice, s);
    }
    if (ce != cudaSuccess)
        return cuda_fail(ce, "cudaMemcpyAsync(intermediate)");
    return MOE_MX_OK;
}

int moe_mx_debug_encode_act(const float *src, int rows, int K, int act_dtype, int method, uint8_t *codes,
                            uint8_t *scale_atoms, void *stream)
{
    g_last_error.clear();
    if (rows < 0 || K < 128 || K % 128 != 0)
        return fail(MOE_MX_ERR_INVALID_ARG, "rows=%d K=%d: need rows >= 0 and K a positive multiple of 128", rows, K);
    if (act_dtype != MOE_MX_ACT_BF16 && act_dtype != MOE_MX_ACT_MXFP8)
        return fail(MOE_MX_ERR_INVALID_ARG, "act_dtype=%d is not MOE_MX_ACT_BF16 or MOE_MX_ACT_MXFP8", act_dtype);
    if (method != 0 && method != 1)
        return fail(MOE_MX_ERR_INVALID_ARG, "method=%d is not 0 or 1", method);
    if (rows == 0)
        return MOE_MX_OK;
    int dev = 0;
    cudaError_t ce = cudaGetDevice(&dev);
    if (ce != cudaSuccess)
        return cuda_fail(ce, "cudaGetDevice");
    int rc;
    if ((rc = check_ptr(src, dev, "src")) || (rc = check_ptr(codes, dev, "codes")) ||
        (rc = check_ptr(scale_atoms, dev, "scale_atoms")))
        return rc;
    int nsm = 148;
    cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    launch_encode_act(src, rows, K, act_dtype == MOE_MX_ACT_MXFP8, method, codes, scale_atoms, nsm,
                      static_cast<cudaStream_t>(stream));
    if ((ce = cudaGetLastError()) != cudaSuccess)
        return cuda_fail(ce, "encoder launch");
    return MOE_MX_OK;
}

long long moe_mx_launch_count(const moe_mx_handle *h) { return h ? h->launches : -1; }

int moe_mx_set_scale_layout(moe_mx_handle *h, int layout)
{
    g_last_error.clear();
    if (!h)
        return fail(MOE_MX_ERR_INVALID_ARG, "handle is NULL");
    if (layout != MOE_MX_SCALES_ROW_MAJOR && layout != MOE_MX_SCALES_TILED)
        return fail(MOE_MX_ERR_INVALID_ARG, "layout=%d is not MOE_MX_SCALES_ROW_MAJOR or MOE_MX_SCALES_TILED", layout);
    h->scale_layout = layout;
    return MOE_MX_OK;
}

int moe_mx_prepare_scales(const moe_mx_handle *h, int which, const uint8_t *src, uint8_t *dst, void *stream)
{
    g_last_error.clear();
    if (!h)
        return fail(MOE_MX_ERR_INVALID_ARG, "handle is NULL");
    if (which != MOE_MX_W1 && which != MOE_MX_W2)
        return fail(MOE_MX_ERR_INVALID_ARG, "which=%d is not MOE_MX_W1 or MOE_MX_W2", which);
    int rc;
    if ((rc = check_ptr(src, h->dev, "src")) || (rc = check_ptr(dst, h->dev, "dst")))
        return rc;
    const int fc1 = which == MOE_MX_W1;
    const int R = fc1 ? 2 * h->I : h->H, K = fc1 ? h->H : h->I;
    const size_t bytes = (size_t)h->E * R * (K / 32);
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(src), a1 = reinterpret_cast<uintptr_t>(dst);
    if (a0 < a1 + bytes && a1 < a0 + bytes)
        return fail(MOE_MX_ERR_INVALID_ARG, "src and dst must not overlap");
    int prev = 0;
    cudaGetDevice(&prev);
    if (prev != h->dev)
        cudaSetDevice(h->dev);
    launch_tile_scales(src, dst, h->E, R, K, fc1, h->num_sms, static_cast<cudaStream_t>(stream));
    cudaError_t ce = cudaGetLastError();
    if (prev != h->dev)
        cudaSetDevice(prev);
    if (ce != cudaSuccess)
        return cuda_fail(ce, "scale tiling launch");
    return MOE_MX_OK;
}

int moe_mx_set_stage_timing(moe_mx_handle *h, int enable)
{
    g_last_error.clear();
    if (!h)
        return fail(MOE_MX_ERR_INVALID_ARG, "handle is NULL");
    int prev = 0;
    cudaGetDevice(&prev);
    cudaSetDevice(h->dev);
    if (h->timing) { // disable, or re-enable = reset
        cudaDeviceSynchronize();
        for (int i = 0; i < kTimingRing * kEvPerFwd; ++i)
            cudaEventDestroy(h->ev[i]);
        delete[] h->ev;
        h->ev = nullptr;
        h->timing = false;
    }
    int rc = MOE_MX_OK;
    if (enable) {
        h->ev = new cudaEvent_t[kTimingRing * kEvPerFwd];
        for (int i = 0; i < kTimingRing * kEvPerFwd; ++i) {
            cudaError_t ce = cudaEventCreate(&h->ev[i]);
            if (ce != cudaSuccess) {
                for (int j = 0; j < i; ++j)
                    cudaEventDestroy(h->ev[j]);
                delete[] h->ev;
                h->ev = nullptr;
                rc = cuda_fail(ce, "cudaEventCreate");
                break;
            }
        }
        if (rc == MOE_MX_OK) {
            h->timing = true;
            h->n_timed = 0;
        }
    }
    cudaSetDevice(prev);
    return rc;
}

int moe_mx_get_stage_times(moe_mx_handle *h, float *ms)
{
    g_last_error.clear();
    if (!h || !ms)
        return fail(MOE_MX_ERR_INVALID_ARG, "handle and ms must be non-NULL");
    if (!h->timing || h->n_timed == 0)
        return fail(MOE_MX_ERR_INVALID_ARG, "stage timing is not enabled or no timed forward ran yet");
    const long long n = h->n_timed < kTimingRing ? h->n_timed : kTimingRing;
    const long long first = h->n_timed - n;
    cudaError_t ce = cudaEventSynchronize(h->ev[((h->n_timed - 1) % kTimingRing) * kEvPerFwd + MOE_MX_NUM_STAGES]);
    if (ce != cudaSuccess)
        return cuda_fail(ce, "cudaEventSynchronize");
    double acc[MOE_MX_NUM_STAGES] = {0};
    for (long long f = first; f < h->n_timed; ++f) {
        cudaEvent_t *set = h->ev + (f % kTimingRing) * kEvPerFwd;
        for (int i = 0; i < MOE_MX_NUM_STAGES; ++i) {
            float v = 0.f;
            if ((ce = cudaEventElapsedTime(&v, set[i], set[i + 1])) != cudaSuccess)
                return cuda_fail(ce, "cudaEventElapsedTime");
            acc[i] += v;
        }
    }
    for (int i = 0; i < MOE_MX_NUM_STAGES; ++i)
        ms[i] = (float)(acc[i] / (double)n);
    return MOE_MX_OK;
}

int moe_mx_debug_watchdog(moe_mx_handle *h, int timeout_us, void *stream)
{
    g_last_error.clear();
    if (!h)
        return fail(MOE_MX_ERR_INVALID_ARG, "handle is NULL");
    if (timeout_us < 1 || timeout_us > 10000000)
        return fail(MOE_MX_ERR_INVALID_ARG, "timeout_us=%d must be in [1, 1e7]", timeout_us);
    launch_watchdog(h->err, (unsigned long long)timeout_us * 1000ull, static_cast<cudaStream_t>(stream));
    cudaError_t ce = cudaGetLastError();
    if (ce != cudaSuccess)
        return cuda_fail(ce, "watchdog launch");
    return MOE_MX_OK;
}

// ---------------------------------------------------------------- routing without allocation
// moe_mx_route_group_noalloc serves callers that cannot allocate device memory
// at the point of the call and keep no handle: a framework op whose device
// memory all comes from the framework's own pool (a cudaMalloc there bypasses
// the pool's accounting and can synchronise the device, stalling every other
// stream), or code that routes once per step from a context where no create /
// destroy lifetime exists.  Its only scratch -- the per-chunk expert
// histograms and the row-block list the grouping kernels write -- lives in the
// file-scope device array below, one copy per device, of fixed size.

} // extern "C"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(1) << 20; // 1 MiB per device

// Nothing in it needs to start at zero: every word a call reads is written
// earlier in the same call (route_kernel writes each chunk's full histogram row
// before scan_kernel reads it).  All calls on one device share it.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxScratchDevices = 64;
std::mutex g_scratch_mu;
void *g_scratch_addr[kMaxScratchDevices]; // per device ordinal, looked up on first use

// Address of this device's copy of the scratch array.  The first lookup on a
// device may load the library's device code there.
int scratch_address(int dev, void **addr)
{
    if (dev < 0 || dev >= kMaxScratchDevices)
        return fail(MOE_MX_ERR_UNSUPPORTED, "device %d is beyond the %d devices the scratch table covers", dev,
                    kMaxScratchDevices);
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        cudaError_t ce = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (ce != cudaSuccess)
            return cuda_fail(ce, "cudaGetSymbolAddress(scratch)");
        g_scratch_addr[dev] = p;
    }
    *addr = g_scratch_addr[dev];
    return MOE_MX_OK;
}

} // namespace

extern "C" {

int moe_mx_route_group_noalloc(const float *router_logits, int num_tokens, int num_experts, int top_k,
                               int32_t *topk_ids, float *topk_w, int32_t *counts, int32_t *pad_offsets,
                               int32_t *sorted_pair, int32_t *pos_of_pair, void *stream)
{
    g_last_error.clear();
    const int T = num_tokens, E = num_experts, k = top_k;
    if (T < 0)
        return fail(MOE_MX_ERR_INVALID_ARG, "num_tokens=%d must be >= 0", T);
    if (E < 1 || E > kMaxExperts)
        return fail(MOE_MX_ERR_UNSUPPORTED, "num_experts=%d must be in [1, %d]", E, kMaxExperts);
    if (k < 1 || k > E || k > kMaxTopK)
        return fail(MOE_MX_ERR_INVALID_ARG, "top_k=%d must be in [1, min(num_experts, %d)]", k, kMaxTopK);
    const int64_t pairs = (int64_t)T * k;
    if (pairs > (int64_t)65536 * kMaxTopK)
        return fail(MOE_MX_ERR_UNSUPPORTED, "num_tokens * top_k = %lld exceeds %lld", (long long)pairs,
                    (long long)65536 * kMaxTopK);
    // scratch plan: [num_rowblocks | pad to 256 B][rowblocks int4 x blocks][chunk histograms int32 x chunks x E]
    auto scratch_bytes = [&](int64_t tokens) {
        const int64_t nchunks = (tokens + kRouteChunk - 1) / kRouteChunk;
        const int64_t nblocks = grouped_rows_bound(E, tokens * k) / kBlockRows;
        return round_up(256 + 16 * nblocks, 256) + 4 * nchunks * E;
    };
    const int64_t off_rowblocks = 256;
    const int64_t off_hist = round_up(off_rowblocks + 16 * (grouped_rows_bound(E, pairs) / kBlockRows), 256);
    if (scratch_bytes(T) > (int64_t)kNoAllocScratchBytes) {
        int64_t lo = 0, hi = T; // largest token count that fits, for the message
        while (lo < hi) {
            const int64_t mid = (lo + hi + 1) / 2;
            if (scratch_bytes(mid) <= (int64_t)kNoAllocScratchBytes)
                lo = mid;
            else
                hi = mid - 1;
        }
        return fail(MOE_MX_ERR_UNSUPPORTED,
                    "num_tokens=%d, num_experts=%d, top_k=%d need %lld bytes of routing scratch; the static "
                    "scratch holds %lld bytes (at most %lld tokens at this expert count and top_k)",
                    T, E, k, (long long)scratch_bytes(T), (long long)kNoAllocScratchBytes, (long long)lo);
    }
    if (T == 0)
        return MOE_MX_OK;
    int dev = 0;
    cudaError_t ce = cudaGetDevice(&dev);
    if (ce != cudaSuccess)
        return cuda_fail(ce, "cudaGetDevice");
    int rc;
    if ((rc = check_ptr(router_logits, dev, "router_logits")) || (rc = check_ptr(topk_ids, dev, "topk_ids")) ||
        (rc = check_ptr(topk_w, dev, "topk_w")) || (rc = check_ptr(counts, dev, "counts")) ||
        (rc = check_ptr(pad_offsets, dev, "pad_offsets")) || (rc = check_ptr(sorted_pair, dev, "sorted_pair")) ||
        (rc = check_ptr(pos_of_pair, dev, "pos_of_pair")))
        return rc;
    void *scratch = nullptr;
    if ((rc = scratch_address(dev, &scratch)))
        return rc;
    unsigned char *base = static_cast<unsigned char *>(scratch);
    RouteGroupArgs ra{router_logits,
                      T,
                      E,
                      k,
                      topk_ids,
                      topk_w,
                      reinterpret_cast<int32_t *>(base + off_hist),
                      counts,
                      pad_offsets,
                      reinterpret_cast<int4 *>(base + off_rowblocks),
                      reinterpret_cast<int32_t *>(base),
                      sorted_pair,
                      pos_of_pair,
                      kBlockRows};
    launch_route_and_group(ra, static_cast<cudaStream_t>(stream));
    ce = cudaGetLastError();
    if (ce != cudaSuccess)
        return cuda_fail(ce, "routing launch");
    return MOE_MX_OK;
}

} // extern "C"
