// route_group.cu -- top-k softmax routing and grouping of (token, slot) pairs
// by expert into the padded grouped layout.
//
// Routing: softmax over the router logits, top-k with the lowest expert index
// winning ties, weights renormalised to sum to 1 (TokenSpeed-kernel README,
// "Public API", moe_route; fusedtok package description, "Operators" and "API
// stability").  The selection is taken on the float32 logits (softmax is
// monotone, so it picks the same experts) which keeps the choice free of exp
// rounding; the k weights are the softmax over the selected logits, which is
// the renormalised full softmax.
//
// Grouping (TokenSpeed-kernel README, "Public API", moe_dispatch): pairs
// p = t*k + j are counting-sorted by expert, stably (ascending t within an
// expert), into segments padded to kBlockRows rows; the activation rows are
// gathered into that order as the MXFP8 operand of the block-scaled FC1 (for
// w4a8 the OCP MXFP8 quantisation of tokenspeed-situ package description,
// "Activation precision (w4a16 vs w4a8)"; for w4a16 an exact two-term
// expansion of the bf16 row).  Every step is deterministic: integer counts only, no float atomics.
#include "kernels.cuh"
#include "ptx.cuh"

namespace moe_mx {

// ---------------------------------------------------------------- router
// Order-preserving map of a float onto uint32 (a < b <=> key(a) < key(b); -0 and +0, which
// compare equal, share a key), and its inverse.
__device__ __forceinline__ uint32_t order_key(float x)
{
    if (x == 0.f)
        x = 0.f;
    const uint32_t u = __float_as_uint(x);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float order_value(uint32_t k)
{
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// Route one token (whole warp): the k experts in descending logit order, the lowest index
// first among equal logits, and their weights = the softmax over the selected logits.  Lane j
// (j < k) writes the j-th id and weight and adds it to the block's expert histogram.
// With n_shared > 0 the token has k + n_shared slots: after the k routed ones, the shared
// expert's chunks (expert slots E.., weight 1).
// With e_local >= 0 the E experts routed over are the whole layer's and this launch holds the
// shard [off, off + e_local) of them: a selected expert inside it is written as its local id
// (global - off) and counted, one outside as -1 (not grouped); the weights are the whole
// layer's, as if unsharded.
template <int kPerLane> // experts per lane: E <= 32 * kPerLane
__device__ __forceinline__ void route_token(const float *__restrict__ row, int E, int k, int n_shared, int t,
                                            int lane, int32_t *__restrict__ topk_ids, float *__restrict__ topk_w,
                                            int32_t *hist, int off = 0, int e_local = -1)
{
    float v[kPerLane];
    uint32_t taken = 0;
#pragma unroll
    for (int i = 0; i < kPerLane; ++i) {
        const int e = i * 32 + lane;
        float x = (e < E) ? __ldg(row + e) : -INFINITY;
        if (x != x) // NaN never outranks a number
            x = -INFINITY;
        v[i] = x;
        if (e >= E)
            taken |= 1u << i; // out of range: never selectable
    }
    // selection j ends up in lane j (k <= 32), so the weights and the writes are lane-parallel
    float my_logit = -INFINITY;
    int my_id = 0;
    for (int j = 0; j < k; ++j) {
        // this lane's best untaken entry (entries are in ascending expert order)
        float bv = -INFINITY;
        int bi = 0x7FFFFFFF;
#pragma unroll
        for (int i = 0; i < kPerLane; ++i) {
            const int e = i * 32 + lane;
            const bool free_ = !((taken >> i) & 1u);
            if (free_ && (v[i] > bv || (v[i] == bv && e < bi))) {
                bv = v[i];
                bi = e;
            }
        }
        // warp arg-max with the lowest index winning ties: the largest value through an
        // order-preserving integer key (one warp reduction), then the lowest index among the
        // lanes holding it (another)
        const uint32_t key = order_key(bv);
        const uint32_t kmax = __reduce_max_sync(0xFFFFFFFFu, key);
        bi = (int)__reduce_min_sync(0xFFFFFFFFu, key == kmax ? (uint32_t)bi : 0xFFFFFFFFu);
        bv = order_value(kmax);
        if ((bi & 31) == lane)
            taken |= 1u << (bi >> 5);
        if (lane == j) {
            my_logit = bv;
            my_id = bi;
        }
    }
    // softmax over the k selected logits == renormalised top-k of the full softmax; the
    // butterfly sum leaves the same z in every lane (each step adds a commutative pair)
    const float m = __shfl_sync(0xFFFFFFFFu, my_logit, 0);
    const float u = lane < k ? expf(my_logit - m) : 0.f;
    float z = u;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
        z += __shfl_xor_sync(0xFFFFFFFFu, z, off);
    const int slots = k + n_shared;
    if (lane < k) {
        const int loc = my_id - off; // off = 0 unless sharded
        const bool local = e_local < 0 || (loc >= 0 && loc < e_local);
        topk_ids[(size_t)t * slots + lane] = local ? loc : -1;
        topk_w[(size_t)t * slots + lane] = u / z;
        if (local)
            atomicAdd(&hist[loc], 1);
    } else if (lane < slots) {
        topk_ids[(size_t)t * slots + lane] = E + (lane - k);
        topk_w[(size_t)t * slots + lane] = 1.0f;
        atomicAdd(&hist[E + (lane - k)], 1);
    }
}

// The given routing of one token (whole warp; lane j takes slot j, k <= 32): global ids mapped
// to the local shard (-1 outside it), weights copied, local experts added to the histogram.
__device__ __forceinline__ void take_given_token(const int32_t *__restrict__ gids, const float *__restrict__ gw,
                                                 int E, int k, int off, int t, int lane,
                                                 int32_t *__restrict__ topk_ids, float *__restrict__ topk_w,
                                                 int32_t *hist)
{
    if (lane < k) {
        const size_t p = (size_t)t * k + lane;
        const int g = __ldg(gids + p);
        const bool local = g >= off && g - off < E; // g >= off >= 0: no overflow in g - off
        topk_ids[p] = local ? g - off : -1;
        topk_w[p] = __ldg(gw + p);
        if (local)
            atomicAdd(&hist[g - off], 1);
    }
}

// One warp per token; each CTA covers kRouteChunk tokens and also writes the
// per-expert histogram of its chunk (the first level of the counting sort).
template <int kPerLane>
__global__ void __launch_bounds__(kRouteThreads) route_kernel(const float *__restrict__ logits, int T, int E,
                                                               int k, int32_t *__restrict__ topk_ids,
                                                               float *__restrict__ topk_w,
                                                               int32_t *__restrict__ chunk_hist,
                                                               const int32_t *__restrict__ gids,
                                                               const float *__restrict__ gw, int off, int n_shared,
                                                               int route_E, int shard)
{
    grid_dep_launch(); // the next kernel (the scan) waits for this grid before reading its output
    grid_dep_wait();   // whatever precedes it (see route_group_small_kernel)
    __shared__ int32_t hist[kMaxExperts];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int e = threadIdx.x; e < E; e += blockDim.x)
        hist[e] = 0;
    __syncthreads();
    const int t_begin = blockIdx.x * kRouteChunk;
    const int t_end = min(T, t_begin + kRouteChunk);
    for (int t = t_begin + warp; t < t_end; t += kRouteThreads / 32) {
        if (gids)
            take_given_token(gids, gw, E, k, off, t, lane, topk_ids, topk_w, hist);
        else
            route_token<kPerLane>(logits + (size_t)t * route_E, route_E, k - n_shared, n_shared, t, lane, topk_ids,
                                  topk_w, hist, off, shard ? E : -1);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x)
        chunk_hist[(size_t)blockIdx.x * E + e] = hist[e];
}

// ---------------------------------------------------------------- scan
// Padded exclusive scan over the experts, for one CTA of 1024 threads (all threads call;
// thread e < E holds its expert's pair count `total`): writes counts, pad_offsets, the
// row-block list and the padding markers, and returns expert e's first grouped row.
// Segments are padded to kBlockRows rows; the row-block list (the GEMMs' work list) splits
// each segment into blocks of at most `split` rows (16, 32, 64 or kBlockRows).
__device__ __forceinline__ int scan_experts(int E, int split, int total, int32_t *__restrict__ counts,
                                            int32_t *__restrict__ pad_offsets, int4 *__restrict__ rowblocks,
                                            int32_t *__restrict__ num_rowblocks, int32_t *__restrict__ sorted_pair,
                                            unsigned long long *s_warp)
{
    const int e = threadIdx.x;
    const int nb = (total + kBlockRows - 1) / kBlockRows; // padded segment: nb * kBlockRows rows
    const int nw = (total + split - 1) / split;            // work blocks of the segment
    // one block-wide exclusive scan of both counts, packed in 32-bit halves
    const unsigned long long mine = ((unsigned long long)nb << 32) | (unsigned)nw;
    unsigned long long incl = mine;
    const int lane = e & 31, warp = e >> 5;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const unsigned long long y = __shfl_up_sync(0xFFFFFFFFu, incl, off);
        if (lane >= off)
            incl += y;
    }
    if (lane == 31)
        s_warp[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        unsigned long long w = s_warp[lane];
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const unsigned long long y = __shfl_up_sync(0xFFFFFFFFu, w, off);
            if (lane >= off)
                w += y;
        }
        s_warp[lane] = w;
    }
    __syncthreads();
    const unsigned long long excl = incl - mine + (warp > 0 ? s_warp[warp - 1] : 0ull);
    const int excl_nb = (int)(excl >> 32), excl_nw = (int)(excl & 0xFFFFFFFFull);
    __shared__ int2 s_pad[kMaxExperts]; // per expert: first padding row, padding rows
    if (e < E) {
        counts[e] = total;
        pad_offsets[e] = excl_nb * kBlockRows;
        if (e == E - 1) {
            pad_offsets[E] = (excl_nb + nb) * kBlockRows;
            *num_rowblocks = excl_nw + nw;
        }
        for (int b = 0; b < nw; ++b)
            rowblocks[excl_nw + b] = make_int4(e, excl_nb * kBlockRows + b * split, min(split, total - b * split), 0);
        s_pad[e] = make_int2(excl_nb * kBlockRows + total, nb * kBlockRows - total);
    }
    __syncthreads();
    // padding markers, one warp per expert: consecutive lanes write consecutive rows (one thread
    // per expert writing its own padding would issue a separate memory transaction per row)
    for (int x = warp; x < E; x += (int)(blockDim.x >> 5)) {
        const int2 pd = s_pad[x];
        for (int r = lane; r < pd.y; r += 32)
            sorted_pair[pd.x + r] = -1;
    }
    return excl_nb * kBlockRows;
}

// One CTA: per-expert totals over the chunk histograms, the scan, and per-chunk base rows
// for the scatter; also zeroes the GEMMs' work-unit counters (optional).  Each expert's chunks
// are split into contiguous ranges over a group of tpe threads (a power of two up to 32, as
// many as 1024 threads allow), so the chunk loop runs tpe-way parallel: the ranges' sums, a
// scan within the group, then (after the expert scan) each range writes its chunks' base rows.
__global__ void __launch_bounds__(1024) scan_kernel(int E, int nchunks, int split, int32_t *__restrict__ chunk_hist,
                                                    int32_t *__restrict__ counts, int32_t *__restrict__ pad_offsets,
                                                    int4 *__restrict__ rowblocks, int32_t *__restrict__ num_rowblocks,
                                                    int32_t *__restrict__ sorted_pair, int32_t *__restrict__ unit_counters)
{
    grid_dep_wait(); // the chunk histograms of the router
    grid_dep_launch();
    __shared__ unsigned long long s_warp[32];
    __shared__ int32_t s_tot[kMaxExperts];
    const int tid = threadIdx.x;
    if (unit_counters && tid < 2) // the GEMMs' work-unit counters start at zero
        unit_counters[tid] = 0;
    int tpe = 1;
    while (tpe < 32 && 2 * tpe * E <= (int)blockDim.x)
        tpe *= 2;
    const int ex = tid / tpe, sub = tid % tpe;
    const bool mine = ex < E;
    const int len = (nchunks + tpe - 1) / tpe;
    const int c_lo = min(nchunks, sub * len), c_hi = min(nchunks, c_lo + len);
    constexpr int kBatch = 16; // loads in flight together
    int part = 0;
    if (mine)
        for (int c0 = c_lo; c0 < c_hi; c0 += kBatch) {
            int h[kBatch];
#pragma unroll
            for (int i = 0; i < kBatch; ++i)
                h[i] = c0 + i < c_hi ? chunk_hist[(size_t)(c0 + i) * E + ex] : 0;
#pragma unroll
            for (int i = 0; i < kBatch; ++i)
                part += h[i];
        }
    // inclusive scan of the ranges within the expert's group of tpe lanes (groups never straddle
    // a warp: tpe divides 32)
    int incl = part;
    for (int off = 1; off < tpe; off <<= 1) {
        const int y = __shfl_up_sync(0xFFFFFFFFu, incl, off);
        if (sub >= off)
            incl += y;
    }
    if (mine && sub == tpe - 1)
        s_tot[ex] = incl;
    __syncthreads();
    const int base = scan_experts(E, split, tid < E ? s_tot[tid] : 0, counts, pad_offsets, rowblocks, num_rowblocks,
                                  sorted_pair, s_warp);
    __syncthreads();
    if (tid < E)
        s_tot[tid] = base; // now: each expert's first grouped row
    __syncthreads();
    if (mine) {
        int run = s_tot[ex] + incl - part; // exclusive prefix within the expert, plus its base row
        for (int c0 = c_lo; c0 < c_hi; c0 += kBatch) {
            int h[kBatch];
#pragma unroll
            for (int i = 0; i < kBatch; ++i)
                h[i] = c0 + i < c_hi ? chunk_hist[(size_t)(c0 + i) * E + ex] : 0;
#pragma unroll
            for (int i = 0; i < kBatch; ++i) {
                if (c0 + i < c_hi)
                    chunk_hist[(size_t)(c0 + i) * E + ex] = run;
                run += h[i];
            }
        }
    }
}

// Stable placement of pairs [p_begin, p_end) by one warp: each pair goes to its expert's
// cursor, pairs in ascending p (so equal experts keep ascending-token order).
__device__ __forceinline__ void scatter_pairs(int p_begin, int p_end, const int32_t *__restrict__ topk_ids,
                                              int32_t *cursor, int32_t *__restrict__ sorted_pair,
                                              int32_t *__restrict__ pos_of_pair, int lane)
{
    const unsigned lt_mask = (1u << lane) - 1u;
    constexpr int kB = 8; // rounds of 32 pairs whose ids are loaded together
    for (int base = p_begin; base < p_end; base += 32 * kB) {
        int ev[kB];
#pragma unroll
        for (int i = 0; i < kB; ++i) {
            const int p = base + 32 * i + lane;
            ev[i] = p < p_end ? topk_ids[p] : -1;
        }
#pragma unroll
        for (int i = 0; i < kB; ++i) {
            if (base + 32 * i >= p_end)
                break; // no pair left in this round (warp-uniform)
            const int p = base + 32 * i + lane;
            const bool valid = p < p_end;
            const bool placed = ev[i] >= 0; // -1: a pair outside the local expert shard (given routing)
            const int e = placed ? ev[i] : -1 - lane; // lanes not placed never match each other
            const unsigned peers = __match_any_sync(0xFFFFFFFFu, e);
            const int rank = __popc(peers & lt_mask);
            int row = 0;
            if (placed)
                row = cursor[e] + rank;
            __syncwarp();
            if (placed && (32 - __clz(peers)) - 1 == lane) // highest lane of the group advances the cursor
                cursor[e] += __popc(peers);
            __syncwarp();
            if (placed) {
                sorted_pair[row] = p;
                pos_of_pair[p] = row;
            } else if (valid) {
                pos_of_pair[p] = -1;
            }
        }
    }
}

// Routing and grouping of a small batch (T <= kSmallRouteTokens) in one CTA: routes, the
// expert histogram, the scan, the row-block list and the stable scatter, with no global
// round trip between the steps.  Also zeroes the GEMMs' work-unit counters.
template <int kPerLane>
__global__ void __launch_bounds__(1024) route_group_small_kernel(const RouteGroupArgs a)
{
    grid_dep_launch(); // the next kernel (the gather) waits for this grid before reading its output
    // Launched as a programmatic dependent of whatever precedes it in the stream (the previous
    // forward's combine, or the caller's kernel that writes the logits): wait for it before
    // reading an input or writing the workspace that kernel may still read.
    grid_dep_wait();
    __shared__ int32_t hist[kMaxExperts]; // counts, then cursors
    __shared__ unsigned long long s_warp[32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int e = threadIdx.x; e < a.E; e += blockDim.x)
        hist[e] = 0;
    if (a.unit_counters && threadIdx.x < 2)
        a.unit_counters[threadIdx.x] = 0;
    for (int i = threadIdx.x; i < a.zero_n; i += blockDim.x)
        a.zero_words[i] = 0;
    __syncthreads();
    for (int t = warp; t < a.T; t += 32) {
        if (a.given_ids)
            take_given_token(a.given_ids, a.given_w, a.E, a.k, a.id_offset, t, lane, a.topk_ids, a.topk_w, hist);
        else
            route_token<kPerLane>(a.logits + (size_t)t * a.routeE(), a.routeE(), a.k - a.n_shared, a.n_shared, t, lane,
                                  a.topk_ids, a.topk_w, hist, a.id_offset, a.shard ? a.E : -1);
    }
    __syncthreads(); // also makes lane 0's id writes visible to the whole CTA
    const int e = threadIdx.x;
    const int total = e < a.E ? hist[e] : 0;
    const int base = scan_experts(a.E, a.split_rows, total, a.counts, a.pad_offsets, a.rowblocks, a.num_rowblocks,
                                  a.sorted_pair, s_warp);
    if (e < a.E)
        hist[e] = base;
    __syncthreads();
    if (warp == 0)
        scatter_pairs(0, a.T * a.k, a.topk_ids, hist, a.sorted_pair, a.pos_of_pair, lane);
}

// ---------------------------------------------------------------- scatter
// One warp per chunk: places the chunk's pairs at their experts' cursors (the chunk's base
// rows from the scan), in ascending p.
__global__ void __launch_bounds__(32) scatter_kernel(int T, int E, int k, const int32_t *__restrict__ topk_ids,
                                                     const int32_t *__restrict__ chunk_base,
                                                     int32_t *__restrict__ sorted_pair,
                                                     int32_t *__restrict__ pos_of_pair)
{
    grid_dep_wait(); // the scan's per-chunk bases (and, through it, the router's ids)
    grid_dep_launch();
    __shared__ int32_t cursor[kMaxExperts];
    const int lane = threadIdx.x;
    for (int e = lane; e < E; e += 32)
        cursor[e] = chunk_base[(size_t)blockIdx.x * E + e];
    __syncwarp();
    const int p_begin = blockIdx.x * kRouteChunk * k;
    const int p_end = min(T, (blockIdx.x + 1) * kRouteChunk) * k;
    scatter_pairs(p_begin, p_end, topk_ids, cursor, sorted_pair, pos_of_pair, lane);
}

// ---------------------------------------------------------------- gather
// Encode each token's row once as the MXFP8 operand FC1 consumes (see mx_encode32): the OCP
// MXFP8 quantisation for w4a8, the exact two-term expansion of the bf16 row for w4a16; and
// write it to the grouped row of `group` of the token's k pairs (group = k: each block is read
// and encoded once; group = 1 for small batches, which need the parallelism more).  One thread
// per (token, 32-element block, pair group): 64 bytes in, group x (32 or 2 x 32) code bytes and
// group x (1 or 2) scale bytes out.
// Codes of one 32-element block, packed four to a word.
// Warp-wide rearrangement of 32 consecutive blocks' codes (lane l holds block l's 32 bytes,
// i.e. 16-byte chunks 2l and 2l + 1 of the warp's 1 KB) so that lane l then holds chunks l and
// l + 32: each 16-byte store instruction of the warp writes 512 contiguous bytes.  Chunk c sits
// at position c ^ ((c >> 3) & 1) of the buffer: no bank conflicts on either side.
__device__ __forceinline__ void transpose_codes(uint4 *stg, int lane, uint4 &lo, uint4 &hi)
{
    const int c0 = 2 * lane, c1 = 2 * lane + 1;
    stg[c0 ^ ((c0 >> 3) & 1)] = lo;
    stg[c1 ^ ((c1 >> 3) & 1)] = hi;
    __syncwarp();
    const int d0 = lane, d1 = lane + 32;
    lo = stg[d0 ^ ((d0 >> 3) & 1)];
    hi = stg[d1 ^ ((d1 >> 3) & 1)];
    __syncwarp();
}

// 32 bf16 values (four 16-byte pieces) as floats.
__device__ __forceinline__ void bf16x32_to_f32(const uint4 (&raw)[4], float (&v)[32])
{
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&raw[i]);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float2 f = __bfloat1622float2(h2[j]);
            v[8 * i + 2 * j] = f.x;
            v[8 * i + 2 * j + 1] = f.y;
        }
    }
}

// At most 128 registers a thread, so that two CTAs (16 warps) share an SM: the kernel streams,
// and its loads need warps in flight to cover their latency.
__global__ void __launch_bounds__(256, 2) gather_kernel(const __nv_bfloat16 *__restrict__ x, int T, int H, int k,
                                                        int group, const int32_t *__restrict__ pos_of_pair,
                                                        uint8_t *__restrict__ aq, uint8_t *__restrict__ asf,
                                                        int act_rows, int act_mxfp8, uint8_t *__restrict__ asf_n,
                                                        int n_rows)
{
    grid_dep_wait(); // pos_of_pair from the grouping
    grid_dep_launch();
    __shared__ __align__(16) uint4 stage[8][2][64]; // per warp and term: 32 blocks' codes
    const int blocks_per_row = H / 32, groups = k / group;
    const long long total = (long long)T * blocks_per_row * groups;
    const long long per_group = (long long)T * blocks_per_row;
    const long long stride = (long long)gridDim.x * blockDim.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (blocks_per_row % 32 == 0) {
        // A warp takes 32 consecutive blocks of one token row (rows are whole multiples of 32
        // blocks, and total a multiple of 32, so every lane has work): the codes of each term go
        // through the warp's buffer once and leave as 512-byte rows per store instruction, to
        // each of the group's grouped rows; the four scale bytes of a 128-element chunk leave as
        // one word from the chunk's first lane.  The x pieces and grouped rows of the warp's next
        // 32 blocks are loaded while it encodes the current ones.
        long long wb = (long long)blockIdx.x * blockDim.x + 32 * warp; // warp-uniform
        uint4 raw[4];
        int my_row = -1; // lane j < group: grouped row of the token's pair jg * group + j
        auto load = [&](long long w) {
            const long long g = w + lane;
            const int jg = (int)(g / per_group);
            const long long tb = g % per_group;
            const int t = (int)(tb / blocks_per_row), b = (int)(tb % blocks_per_row);
            const uint4 *src = reinterpret_cast<const uint4 *>(x + (size_t)t * H + (size_t)b * 32);
#pragma unroll
            for (int i = 0; i < 4; ++i)
                raw[i] = __ldg(src + i);
            my_row = lane < group ? pos_of_pair[(size_t)t * k + jg * group + lane] : -1;
        };
        if (wb < total)
            load(wb);
        for (; wb < total; wb += stride) {
            const long long tb = (wb + lane) % per_group;
            const int b = (int)(tb % blocks_per_row);
            const int b0 = b - lane; // the warp's first block
            float v[32];
            bf16x32_to_f32(raw, v);
            const int rows_now = my_row;
            if (wb + stride < total)
                load(wb + stride);
            uint32_t c0[8], c1[8];
            uint32_t s0, s1;
            mx_encode32(v, act_mxfp8, c0, c1, s0, s1); // the values are bf16 already: no rounding step
            uint4 a_lo = make_uint4(c0[0], c0[1], c0[2], c0[3]), a_hi = make_uint4(c0[4], c0[5], c0[6], c0[7]);
            uint4 b_lo = make_uint4(c1[0], c1[1], c1[2], c1[3]), b_hi = make_uint4(c1[4], c1[5], c1[6], c1[7]);
            transpose_codes(stage[warp][0], lane, a_lo, a_hi);
            if (!act_mxfp8)
                transpose_codes(stage[warp][1], lane, b_lo, b_hi);
            // the scale bytes of blocks 4m .. 4m + 3 (one 128-element chunk) as one word
            uint32_t w0 = s0, w1 = s1;
#pragma unroll
            for (int i = 1; i < 4; ++i) {
                w0 |= __shfl_down_sync(0xFFFFFFFFu, s0, i) << (8 * i);
                w1 |= __shfl_down_sync(0xFFFFFFFFu, s1, i) << (8 * i);
            }
            for (int j = 0; j < group; ++j) {
                const int row = __shfl_sync(0xFFFFFFFFu, rows_now, j); // the same for the whole warp
                if (row < 0)
                    continue; // not in the local expert shard
                uint4 *dst = reinterpret_cast<uint4 *>(aq + (size_t)row * H + (size_t)b0 * 32);
                dst[lane] = a_lo;
                dst[lane + 32] = a_hi;
                if ((lane & 3) == 0) {
                    *reinterpret_cast<uint32_t *>(asf + sf_atom_byte(row, b * 32, H, 0)) = w0;
                    if (asf_n)
                        *reinterpret_cast<uint32_t *>(asf_n + sf_n_byte(row, b * 32, H, 0, n_rows)) = w0;
                }
                if (!act_mxfp8) {
                    uint4 *dst1 = reinterpret_cast<uint4 *>(aq + ((size_t)act_rows + row) * H + (size_t)b0 * 32);
                    dst1[lane] = b_lo;
                    dst1[lane + 32] = b_hi;
                    if ((lane & 3) == 0) {
                        *reinterpret_cast<uint32_t *>(asf + sf_atom_byte(row, b * 32, H, 1)) = w1;
                        if (asf_n)
                            *reinterpret_cast<uint32_t *>(asf_n + sf_n_byte(row, b * 32, H, 1, n_rows)) = w1;
                    }
                }
            }
        }
        return;
    }
    for (long long g = blockIdx.x * (long long)blockDim.x + threadIdx.x; g < total; g += stride) {
        // consecutive threads take consecutive blocks of one row: coalesced loads and stores
        const int jg = (int)(g / per_group);
        const long long tb = g % per_group;
        const int t = (int)(tb / blocks_per_row);
        const int b = (int)(tb % blocks_per_row);
        const uint4 *src = reinterpret_cast<const uint4 *>(x + (size_t)t * H + (size_t)b * 32);
        uint4 raw[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            raw[i] = __ldg(src + i);
        float v[32];
        bf16x32_to_f32(raw, v);
        uint32_t c0[8], c1[8];
        uint32_t s0, s1;
        mx_encode32(v, act_mxfp8, c0, c1, s0, s1); // the values are bf16 already: no rounding step
        for (int j = jg * group; j < (jg + 1) * group; ++j) {
            const int row = pos_of_pair[(size_t)t * k + j];
            if (row < 0)
                continue; // not in the local expert shard
            store_codes32(aq + (size_t)row * H + b * 32, c0);
            asf[sf_atom_byte(row, b * 32, H, 0)] = (uint8_t)s0;
            if (asf_n)
                asf_n[sf_n_byte(row, b * 32, H, 0, n_rows)] = (uint8_t)s0;
            if (!act_mxfp8) {
                store_codes32(aq + ((size_t)act_rows + row) * H + b * 32, c1);
                asf[sf_atom_byte(row, b * 32, H, 1)] = (uint8_t)s1;
                if (asf_n)
                    asf_n[sf_n_byte(row, b * 32, H, 1, n_rows)] = (uint8_t)s1;
            }
        }
    }
}

// ---------------------------------------------------------------- combine
// out[t, n] = bf16( sum_{j<k} w[t,j] * Y[pos(t,j), n] ), j ascending, f32.
// Y is kept in f32 so the only rounding of the result is the final one.
// One thread per 8 consecutive outputs (2 x 16-byte loads per slot, one 16-byte store).
template <bool kOutF32>
__global__ void __launch_bounds__(256) combine_kernel(const float *__restrict__ Y, int T, int H, int k,
                                                      const int32_t *__restrict__ pos_of_pair,
                                                      const float *__restrict__ topk_w, void *__restrict__ out)
{
    grid_dep_wait(); // Y from FC2
    const int vec_per_row = H / 8;
    const long long total = (long long)T * vec_per_row;
    for (long long g = blockIdx.x * (long long)blockDim.x + threadIdx.x; g < total;
         g += (long long)gridDim.x * blockDim.x) {
        const int t = (int)(g / vec_per_row);
        const int c = (int)(g % vec_per_row);
        float acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
            acc[i] = 0.f;
        for (int j = 0; j < k; ++j) {
            const float w = __ldg(topk_w + (size_t)t * k + j);
            const int row = __ldg(pos_of_pair + (size_t)t * k + j);
            if (row < 0)
                continue; // a pair outside the local expert shard: no contribution
            const float4 *src = reinterpret_cast<const float4 *>(Y + (size_t)row * H) + 2 * c;
            const float4 a0 = __ldg(src), a1 = __ldg(src + 1);
            acc[0] = fmaf(w, a0.x, acc[0]);
            acc[1] = fmaf(w, a0.y, acc[1]);
            acc[2] = fmaf(w, a0.z, acc[2]);
            acc[3] = fmaf(w, a0.w, acc[3]);
            acc[4] = fmaf(w, a1.x, acc[4]);
            acc[5] = fmaf(w, a1.y, acc[5]);
            acc[6] = fmaf(w, a1.z, acc[6]);
            acc[7] = fmaf(w, a1.w, acc[7]);
        }
        if (kOutF32) {
            // a shard's partial output, kept in float32 for the sum over shards
            float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(out) + (size_t)t * H) + 2 * c;
            dst[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
            dst[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
        } else {
            uint4 o;
            __nv_bfloat162 *o2 = reinterpret_cast<__nv_bfloat162 *>(&o);
#pragma unroll
            for (int i = 0; i < 4; ++i)
                o2[i] = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
            reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(out) + (size_t)t * H)[c] = o;
        }
    }
}

// ---------------------------------------------------------------- launchers
int launch_route_and_group(const RouteGroupArgs &a, cudaStream_t s, bool pdl)
{
    // the top-k scan visits 32 * kPerLane candidates per token: size it to the expert count
    // (the given routing visits no candidates: the smallest instance serves it).  With pdl every
    // kernel is a programmatic dependent of the one before it in the stream, the first one too
    // (its launch overlaps the tail of whatever precedes it; it waits for that before its work).
    const bool narrow = a.given_ids != nullptr || a.routeE() <= 256;
    if (a.T <= kSmallRouteTokens) {
        if (narrow)
            launch_kernel(route_group_small_kernel<8>, dim3(1), dim3(1024), 0, s, pdl, a);
        else if (a.routeE() <= 512)
            launch_kernel(route_group_small_kernel<16>, dim3(1), dim3(1024), 0, s, pdl, a);
        else
            launch_kernel(route_group_small_kernel<32>, dim3(1), dim3(1024), 0, s, pdl, a);
        return 1;
    }
    const int nchunks = (a.T + kRouteChunk - 1) / kRouteChunk;
    auto route = [&](auto kernel) {
        launch_kernel(kernel, dim3(nchunks), dim3(kRouteThreads), 0, s, pdl, a.logits, a.T, a.E, a.k, a.topk_ids,
                      a.topk_w, a.chunk_hist, a.given_ids, a.given_w, a.id_offset, a.n_shared, a.routeE(), a.shard);
    };
    if (narrow)
        route(route_kernel<8>);
    else if (a.routeE() <= 512)
        route(route_kernel<16>);
    else
        route(route_kernel<32>);
    launch_kernel(scan_kernel, dim3(1), dim3(1024), 0, s, pdl, a.E, nchunks, a.split_rows, a.chunk_hist, a.counts,
                  a.pad_offsets, a.rowblocks, a.num_rowblocks, a.sorted_pair, a.unit_counters);
    launch_kernel(scatter_kernel, dim3(nchunks), dim3(32), 0, s, pdl, a.T, a.E, a.k, (const int32_t *)a.topk_ids,
                  (const int32_t *)a.chunk_hist, a.sorted_pair, a.pos_of_pair);
    return 3;
}

void launch_gather(const __nv_bfloat16 *x, int P, int H, int k, const int32_t *pos_of_pair, uint8_t *aq,
                   uint8_t *asf, int act_rows, int act_mxfp8, uint8_t *asf_n, int n_rows, int num_sms,
                   cudaStream_t s, bool pdl)
{
    // encode each block once per token when that still fills the GPU, else once per pair
    const long long token_blocks = (long long)(P / k) * (H / 32);
    const int group = token_blocks >= (long long)num_sms * 1024 ? k : 1;
    const long long work = token_blocks * (k / group);
    const long long want = (work + 255) / 256;
    const int grid = (int)(want < (long long)num_sms * 8 ? want : (long long)num_sms * 8);
    launch_kernel(gather_kernel, dim3(grid > 0 ? grid : 1), dim3(256), 0, s, pdl, x, P / k, H, k, group, pos_of_pair,
                  aq, asf, act_rows, act_mxfp8, asf_n, n_rows);
}

void launch_combine(const float *Y, int T, int H, int k, const int32_t *pos_of_pair, const float *topk_w, void *out,
                    int out_f32, int num_sms, cudaStream_t s, bool pdl)
{
    const long long work = (long long)T * (H / 8);
    const long long want = (work + 255) / 256;
    const int grid = (int)(want < (long long)num_sms * 8 ? want : (long long)num_sms * 8);
    launch_kernel(out_f32 ? combine_kernel<true> : combine_kernel<false>, dim3(grid > 0 ? grid : 1), dim3(256), 0, s,
                  pdl, Y, T, H, k, pos_of_pair, topk_w, out);
}

} // namespace moe_mx
