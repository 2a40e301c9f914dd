// fc_gemm.cu -- persistent grouped GEMM for FC1 (+SwiGLU) and FC2 on the
// 5th-generation tensor cores, consuming the MXFP4 weights directly.
//
// What it computes (tokenspeed-situ package description, intro: FC1 "MXFP4 +
// <gated activation>" and the matching FC2, and "Activation precision (w4a16
// vs w4a8)"): for every row block (an expert's slice of at most 128 grouped
// rows) and every 128-row tile of that expert's weight,
//     D[rows, 128] = A[rows, K] . W[128, K]^T,   f32 accumulation,
// with W the E2M1 codes times their E8M0 block scales (OCP MX: one scale per 32
// elements along K) and A the activation rows as MXFP8 E4M3 with E8M0 block
// scales.  tcgen05.mma kind::mxf8f6f4.block_scale applies both scales inside
// the tensor core, so no weight element is ever dequantised by the ALU:
//   * w4a8: A is the MXFP8-quantised activation (one term);
//   * w4a16: A is a two-term MXFP8 expansion of the bf16 activation,
//     x = x1 + x2 (see mx_encode32 in kernels.cuh), accumulated by two MMAs
//     into the same TMEM accumulator.
// FC1 tiles hold 64 gate rows followed by the matching 64 up rows, so the
// epilogue forms h = silu(gate) * up and writes h for FC2 in the same MXFP8
// form (two terms of h rounded to bf16 for w4a16; the OCP-quantised h for
// w4a8, whose dequantised value is the bf16 value FC2 consumes).  FC2 writes
// f32 rows that the combine kernel sums.
//
// Per CTA (one per SM, persistent; work units u = (row block, weight tile) handed
// out at run time through a global counter):
//   producers   2 to 4 warps, taking pipeline stages round robin (in pairs in
//               the weight-streaming variants): TMA of the weight tile (E2M1
//               codes unpacked to 8-bit containers; for FC1 the gate and up
//               halves in one 3-D box), TMA of both activation term planes in
//               one 3-D box, the stage's weight scale atom (one bulk copy in the
//               tiled layout, else 4-byte copies) and the activation scale atom
//               (bulk copy; with the tokens on N 4-byte copies laid out for N,
//               or, in the kScalesN kernels, one bulk copy of the atom the
//               activations' producer wrote in that N layout);
//   MMA         1 or 2 warps (alternate stages, own accumulators): tcgen05.cp of
//               the stage's scale atoms to TMEM, then the block-scaled MMAs; one
//               warp owns the TMEM allocation;
//   epilogue    4 warps (tcgen05.ld); accumulators double-buffered in TMEM;
//   scheduler   1 warp: claims work units and publishes them (with their row
//               block) in a small shared-memory ring every other warp reads.
// Orientation per work unit: a block of more than `swap_rows` rows puts its
// tokens on the MMA's M side (M = 128, N = 128 weight rows); a smaller block
// (decode) puts the weight rows on M and its tokens on N (16..128), so the
// tensor core does not multiply padding rows.  With the tokens on N, the two
// w4a16 terms sit side by side on N as well (term 2 from column kT2 on), so one
// MMA per 32-element K block covers both: an M = 128 block-scaled MMA occupies
// the tensor pipe about as long for N = 16 as for N = 128 (measured), so this
// halves the pipe time of the weight-streaming shapes.  A work unit takes 1, 2 or 4
// adjacent weight tiles (4 only with tokens on N at up to 16 rows, where four
// 32-column accumulators share a 128-column TMEM buffer): fewer, larger stages
// keep more weight bytes in flight per SM.
// One launch may also run two phases (kTwo): FC1's units, then FC2's, claimed from
// one counter; FC1's epilogue counts each row block's finished units and an FC2
// unit's producers wait for that count before copying h.  Every wait is bounded;
// a wait that gives up records an error word, and the CTA drains its own copies
// and MMAs before freeing TMEM.
#include "kernels.cuh"
#include "ptx.cuh"

namespace moe_mx {

namespace {

constexpr int kTermRowBytes = 128;             // one activation row of a K stage: 128 E4M3 codes
constexpr int kWBytes = 128 * 128;             // 128 rows x 128 E2M1 codes in 8-bit containers
constexpr int kWTxBytes = 128 * 128 / 2;       // ... of which the TMA transfers (and counts) the packed 4-bit data
constexpr int kAsfBytes = 2 * 512;             // one 512-byte scale atom per term
constexpr int kWsfBytes = 512;
constexpr int kXBytes = 64 * 16 * 4;           // epilogue exchange, 64 lanes x 16 columns f32
constexpr int kSmemLimit = 227 * 1024;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSfCol = 256; // TMEM columns 256..267 hold the stage's scale factors
constexpr unsigned long long kDrainTimeoutNs = 200000000ull;
// Work units are handed out at run time (a global counter): SMs do not all stream at the same
// rate (measured: up to 25 % apart on the same work), so a fixed round-robin share leaves the
// kernel waiting on the slowest.  A scheduler warp takes the CTA's next units from the counter
// and publishes them through a ring of kRing slots in shared memory; a slot is refilled once
// every reading warp has taken it, which keeps the claims a few units ahead of the work.
constexpr int kRing = 4;

// Shared-memory plan for a kernel whose activation tiles hold at most kActRows
// rows per term: as many pipeline stages as fit (more stages = more bytes in
// flight per SM, which is what the weight-streaming decode shapes need).
template <int kActRows, int kMmaW, int kWTiles, int kTm> struct Plan {
    // first N row of the second activation term when both terms share one MMA (tokens on N)
    static constexpr int kT2 = kActRows < 64 ? kActRows : 64;
    static constexpr int kTermBytes = kActRows * kTermRowBytes;
    // activation term planes a stage holds: 2 (the w4a16 split; any launch), or 1 for the
    // variant that only takes single-term launches (w4a8 FC1), whose smaller stages leave room
    // for more of them
    static_assert(kTm == 1 || kTm == 2, "activation terms per stage");
    static constexpr int kActBytes = kTm * kTermBytes;
    // weight tiles per work unit (1, or 2 adjacent 128-row tiles against one activation block:
    // twice the weight bytes per stage for the same per-stage bookkeeping and activation copy)
    static constexpr int kWT = kWTiles;
    static constexpr int kWStage = kWT * kWBytes, kWsfStage = kWT * kWsfBytes;
    static constexpr int kStageBytes = kActBytes + kWStage + kAsfBytes + kWsfStage;
    // wide variant: a 2 KB staging buffer per epilogue warp for FC2's f32 output rows
    static constexpr int kYBytes = (kActRows == 128 && kWTiles == 2) ? 8 * 2048 : 0;
    static constexpr int kStages = (kSmemLimit - 1024 - kXBytes - kYBytes - 256) / kStageBytes;
    // The per-stage copy issue is split over several producer warps: each TMA instruction and
    // each warp-wide 4-byte scale copy occupies its issuing warp for about a hundred cycles
    // (measured: the cost is per warp, not per SM).  Measured on the 16-row FC1 at decode: 2
    // producer warps 25 % slower than 4, and 6 slower still (70 %), with producers then
    // sharing the MMA warps' schedulers.  With single stages round robin a producer's
    // consecutive stages are kProd apart; its parity waits on a slot's "empty" barrier are
    // only sound while it cannot get two rounds ahead of that slot, which holds when
    // kProd <= kStages.
    static constexpr int kProdWant = kActRows < 128 ? 4 : 2;
    static constexpr int kProd = kProdWant <= kStages ? kProdWant : kStages;
    static_assert(kProd >= 1 && kProd <= kStages, "producer warps vs pipeline stages");
    // Weight-streaming variants hand out stages in pairs (2m, 2m + 1 to producer m % kProd): a
    // K stage holds 64 bytes of each packed weight row, so one warp then requests both halves of
    // a row's 128-byte line back to back (measured: batched decode FC1 0.971 -> 0.954 ms).
    // Soundness of a producer's parity wait for stage g (slot g % kStages): it passes early only
    // if stage g - 2 kStages is still unconsumed.  By induction the producer's own earlier
    // stages g' were issued after stage g' - kStages was consumed.  With one MMA warp stages are
    // consumed in order, and its previous stage is at least g - (2 kProd - 1), which rules the
    // early pass out when 2 kProd - 1 <= kStages.  With two MMA warps (one per stage parity,
    // each in order, kStages even) the producer's previous pair holds a stage of g's parity at
    // least g - 2 kProd: 2 kProd <= kStages.
    static constexpr bool kPairStages =
        kActRows < 128 && (kMmaW == 1 ? 2 * kProd - 1 <= kStages : 2 * kProd <= kStages);
    // single stages round robin with two MMA warps: the producer's previous stage of g's parity
    // is g - kProd (kProd even) or g - 2 kProd
    static_assert(kMmaW == 1 || kPairStages || kProd % 2 == 0 || 2 * kProd <= kStages,
                  "producer parity waits with two MMA warps");
    // producer role index of stage g
    static __device__ __forceinline__ int producer_of(uint32_t g)
    {
        return (int)((kPairStages ? (g >> 1) : g) % (uint32_t)kProd);
    }
    // With at most 32 tokens per block (N <= 64) two MMA warps may take alternate stages,
    // each into its own accumulator (the epilogue adds them): one thread issues a block-scaled
    // MMA about every 64 cycles, and the second warp hides the per-stage wait and bookkeeping.
    // (Measured: a gain for FC1's long units, a loss for FC2's short ones; the launch chooses.)
    // (Each MMA warp waits on the stages of its own parity only, and kStages is even, so its
    // parity waits on "full" barriers are never two phases ahead either.)
    static constexpr int kMma = kMmaW;
    static_assert(kMma == 1 || kStages % 2 == 0, "alternating MMA warps need an even stage count");
    static_assert(kMma == 1 || kActRows <= 32, "two accumulators per buffer need N <= 64");
    static_assert(kWT == 1 || (kWT == 2 && kMma == 1 && (kActRows <= 32 || kActRows == 128)) ||
                      (kWT == 4 && kMma == 1 && kActRows <= 16),
                  "two weight tiles: one MMA warp, N <= 64 or the wide 128-row variant; four: N <= 32");
    // TMEM columns between the accumulators of a unit's weight tiles within one 128-column buffer:
    // 64, or 32 for four tiles (N <= 32)
    static constexpr int kAccW = kWT == 4 ? 32 : 64;
    // The wide variant (128 token rows against two weight tiles, tokens on M): one M = 128,
    // N = 256 MMA per K block covers both tiles, so each activation byte brought into shared
    // memory feeds twice the MMA work.  Its 256-column accumulator leaves no room in TMEM for a
    // second one beside the scale factors, so it is single-buffered; 8 epilogue warps (two per
    // TMEM lane quarter, one per tile) copy it to registers and release it at once.
    static constexpr bool kWide = kActRows == 128 && kWT == 2;
    static constexpr int kEpiWarps = kWide ? 8 : 4;
    // warps: producer 0, MMA 0, 4 epilogue, producers 1.., MMA 1 (if any), 4 more epilogue
    // (wide), the scheduler
    static constexpr int kEpi2 = 5 + kProd + (kMma - 1); // first warp of the second epilogue group
    static constexpr int kThreads = 32 * (2 + kEpiWarps + (kProd - 1) + (kMma - 1) + 1);
    static constexpr int kOffAct = 0;
    static constexpr int kOffW = kOffAct + kStages * kActBytes;
    static constexpr int kOffAsf = kOffW + kStages * kWStage;
    static constexpr int kOffWsf = kOffAsf + kStages * kAsfBytes;
    static constexpr int kOffX = kOffWsf + kStages * kWsfStage;
    static constexpr int kOffY = kOffX + kXBytes;
    static constexpr int kOffBar = kOffY + kYBytes;
    static constexpr int kNumBars = 2 * kStages + 1 + 4 + 2 * kRing;
    static constexpr int kOffTmemSlot = kOffBar + kNumBars * 8;
    static constexpr int kOffUnits = kOffTmemSlot + 16;                 // the work-unit ring
    static constexpr int kSmemBytes = kOffUnits + 16 * kRing + 1024;   // + slack for 1024-byte alignment
    static_assert(kSmemBytes <= kSmemLimit, "shared memory plan too large");
    static_assert(kStages >= 3, "too few pipeline stages");
};

constexpr uint32_t kFmtE4M3 = 0, kFmtE2M1 = 5;

template <int kStages> struct Bars {
    uint32_t base;
    __device__ uint32_t full(int s) const { return base + 8 * s; }
    __device__ uint32_t empty(int s) const { return base + 8 * (kStages + s); }
    __device__ uint32_t mma_done() const { return base + 8 * (2 * kStages); }
    __device__ uint32_t acc_full(int b) const { return base + 8 * (2 * kStages + 1 + b); }
    __device__ uint32_t acc_empty(int b) const { return base + 8 * (2 * kStages + 3 + b); }
    __device__ uint32_t ring_full(int i) const { return base + 8 * (2 * kStages + 5 + i); }
    __device__ uint32_t ring_empty(int i) const { return base + 8 * (2 * kStages + 5 + kRing + i); }
};

// Readers of the work-unit ring: every producer and MMA warp and each of the 4 epilogue warps
// reads every slot, then releases it.
// A slot holds the unit's row block {expert, first grouped row, rows} and, in .w, the unit
// index (-1: no more work), so that no reader has to fetch the row block from global memory.
template <int kStages> struct UnitRing {
    Bars<kStages> bars;
    volatile int *slots; // kRing x 4 ints
    // The CTA's i-th work unit (.w = -1: no more work, or a wait gave up).  Whole warp.
    __device__ int4 take(uint32_t i, uint32_t *err, unsigned long long tmo, int lane) const
    {
        const int r = (int)(i % kRing);
        int4 v = make_int4(0, 0, 0, -1);
        if (__all_sync(0xFFFFFFFFu, mbar_wait_bounded(bars.ring_full(r), (i / kRing) & 1, err, tmo)))
            v = make_int4(slots[4 * r], slots[4 * r + 1], slots[4 * r + 2], slots[4 * r + 3]);
        __syncwarp();
        if (lane == 0)
            mbar_arrive(bars.ring_empty(r));
        return v;
    }
    // Scheduler (one lane): publish the CTA's j-th unit; false once the work is exhausted.  Units
    // [0, units0) belong to phase 0 (n_groups0 per row block), the rest to phase 1.
    __device__ bool fill(uint32_t j, const FcGemmArgs &a, int total_units, int units0, int n_groups0,
                         int n_groups1, unsigned long long tmo) const
    {
        const int r = (int)(j % kRing);
        const bool got = mbar_wait_bounded(bars.ring_empty(r), ((j / kRing) & 1) ^ 1, a.err, tmo);
        int u = got ? atomicAdd(a.unit_counter, 1) : -1;
        int4 blk = make_int4(0, 0, 0, 0);
        if (u >= total_units)
            u = -1;
        if (u >= 0)
            blk = a.rowblocks[u < units0 ? u / n_groups0 : (u - units0) / n_groups1];
        slots[4 * r] = blk.x;
        slots[4 * r + 1] = blk.y;
        slots[4 * r + 2] = blk.z;
        slots[4 * r + 3] = u;
        mbar_arrive(bars.ring_full(r)); // release: the slot writes are seen by every reader's acquire
        return u >= 0;
    }
};

// One lane of a converged warp is elected (tcgen05 and TMA instructions are
// issued once per warp while the whole warp runs the loop, so their operands
// stay warp-uniform).
__device__ __forceinline__ bool elect_one()
{
    uint32_t p = 0;
    asm volatile("{\n\t.reg .pred P;\n\telect.sync _|P, 0xffffffff;\n\tselp.b32 %0, 1, 0, P;\n\t}" : "=r"(p));
    return p != 0;
}

// Instruction descriptor of kind::mxf8f6f4 with E8M0 block scales (one scale
// per 32 elements): [4,6) B scale byte, [7,10) A format, [10,13) B format,
// [17,23) N/8, [23] scale format E8M0, [24,29) M/16, [29,31) A scale byte.
__device__ __forceinline__ uint32_t idesc_mx(uint32_t a_fmt, uint32_t b_fmt, uint32_t M, uint32_t N, uint32_t sf_id)
{
    return (sf_id << 4) | (a_fmt << 7) | (b_fmt << 10) | ((N >> 3) << 17) | (1u << 23) | ((M >> 4) << 24) |
           (sf_id << 29);
}

__device__ __forceinline__ void umma_mx(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
        : "memory");
}

// Copy one 512-byte scale atom (32 rows x 16 bytes) from shared memory to TMEM
// columns [col, col+4), replicated into the four 32-lane quarters: lane
// (32q + r) column (col + j) then holds the four scale bytes (one per 32-element
// block) of tile row r + 32j.
__device__ __forceinline__ void tmem_cp_sf_atom(uint32_t taddr, uint32_t saddr)
{
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFF);
    d |= (uint64_t)1 << 16;          // leading offset (single 16-byte column)
    d |= (uint64_t)(128 >> 4) << 32; // next 8-row core matrix: 128 bytes
    d |= (uint64_t)1 << 46;          // descriptor version
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(d) : "memory");
}

__device__ __forceinline__ void bulk_copy_g2s(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     dst),
                 "l"(src), "r"(bytes), "r"(bar)
                 : "memory");
}

__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t count)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// All `count` threads of named barrier `id` agree on v (logical AND).
__device__ __forceinline__ bool named_bar_all(uint32_t id, uint32_t count, bool v)
{
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "barrier.cta.red.and.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v), "r"(id), "r"(count)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ float silu_mul(float g, float u)
{
    return g / (1.0f + expf(-g)) * u;
}

} // namespace


// The combine fused into FC2's epilogue (small batches, every unit with its tokens on N), run by
// the 128 epilogue threads (L = 0..127) after a unit's Y rows are stored.  Each (token, weight
// tile) those rows belong to counts one more finished pair; the unit that completes a token's k
// pairs of a tile sums the token's k rows of that tile in j order, out = bf16(sum_j w_j * Y_j)
// with the combine kernel's arithmetic (same bits), and resets the count for the next forward.
// Every Y store is fenced before its count, and the completing unit fences before it reads.
__device__ __forceinline__ void fused_combine_unit(const FcGemmArgs &a, const int4 blk, int nt0, int kWT, int L,
                                                   int *s_list)
{
    __threadfence();
    if (L == 0)
        s_list[128] = 0;
    named_bar_sync(1, 128);
    if (L < blk.z * kWT) { // one (row, weight tile) per thread: rows <= 64, kWT <= 2
        const int n = L / kWT, tile = nt0 + L % kWT;
        const int t = a.sorted_pair[blk.y + n] / a.k;
        int *c = a.combine_cnt + (size_t)t * a.n_tiles + tile;
        if (atomicAdd(c, 1) == a.k - 1) {
            *c = 0; // the token's last pair of this tile: nothing else counts it in this forward
            s_list[atomicAdd(&s_list[128], 1)] = t * a.n_tiles + tile;
        }
    }
    named_bar_sync(1, 128);
    __threadfence();
    const int ne = s_list[128];
    for (int i = 0; i < ne; ++i) {
        const int t = s_list[i] / a.n_tiles, col = (s_list[i] % a.n_tiles) * 128 + L;
        float acc = 0.f;
        for (int j = 0; j < a.k; ++j) {
            const float w = __ldg(a.topk_w + (size_t)t * a.k + j);
            const int row = __ldg(a.pos_of_pair + (size_t)t * a.k + j);
            acc = fmaf(w, __ldcg(a.y + (size_t)row * a.out_ld + col), acc);
        }
        a.out[(size_t)t * a.out_ld + col] = __float2bfloat16_rn(acc);
    }
    named_bar_sync(1, 128); // the list is rewritten by the next unit
}

// Per-CTA state the warp roles share (all values are CTA-uniform).  A launch runs one phase (one
// GEMM) or two (FC1's units, then FC2's): per phase its arguments, tensor maps, work units per
// row block (tile groups), K stages and activation terms; a unit's phase follows from its index.
struct Ctx {
    uint32_t base;        // shared-memory base (1024-byte aligned, shared window)
    volatile int *units;  // the work-unit ring (generic pointer to shared memory)
    uint8_t *ystage;      // wide variant: the epilogue warps' FC2 staging buffers (shared memory)
    uint32_t tmem_base;
    int total_units, units0; // all units; those of phase 0 (units0 == total_units: one phase)
    const FcGemmArgs *args[2];
    const CUtensorMap *maps[2][4]; // act_map, act_map_sw, act_map16, w_map
    int n_groups[2], kst[2], terms[2];
    unsigned long long tmo;
    uint32_t *err;
    bool two; // a compile-time constant of the kernel (kTwo): one-phase kernels fold every phase to 0
    __device__ int phase(int u) const { return two && u >= units0 ? 1 : 0; }
    __device__ int local(int u) const { return two && u >= units0 ? u - units0 : u; } // index within its phase
};

// Bounded wait (one thread) until *count >= target, read with acquire semantics at GPU scope, then
// a proxy fence so that the caller's later TMA reads (async proxy) see what the counted writers
// stored before counting.  False (and the error word set) if the limit ran out.
__device__ __forceinline__ bool wait_count(const int32_t *count, int target, uint32_t *err,
                                           unsigned long long timeout_ns)
{
    const long long t0 = clock64();
    for (uint32_t it = 0;; ++it) {
        int v;
        asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(count) : "memory");
        if (v >= target)
            break;
        if ((it & 63) == 63) {
            const unsigned long long dt = (unsigned long long)(clock64() - t0);
            if (dt > 100000ull && *(volatile uint32_t *)err != 0)
                return false;
            if (dt > timeout_ns) {
                atomicOr(err, kErrTimeout);
                return false;
            }
        }
    }
    asm volatile("fence.proxy.async.global;" ::: "memory");
    return true;
}

// Producer role, one of kProd warps taking the stages g with Plan::producer_of(g) == PI (PI is
// a compile-time role index so that every operand of the TMA issue stays warp-uniform): stage
// pairs in the weight-streaming variants, so that the two 64-byte halves of a weight row's
// 128-byte line are requested together, else single stages round robin.
// Launched as a programmatic dependent, the kernel may start while the kernel ahead of it (which
// writes this GEMM's activations) still runs; the producers wait for it (grid_dep_wait) before
// their first copy.  (Issuing the first pass's weight copies before that wait and deferring only
// the activation copies measured slower: the extra paths cost the steady-state loop more than
// the early weights gained.)
template <int kActRows, int kMmaW, int kWTiles, int kTm, int PI, bool kScalesN>
__device__ __forceinline__ void producer_role(const Ctx &c, int lane)
{
    uint32_t *const err_w = c.err; // in a register: the stage loops wait with it
    using P = Plan<kActRows, kMmaW, kWTiles, kTm>;
    constexpr int kStages = P::kStages, kProd = P::kProd, kWT = P::kWT;
    constexpr int kTermBytes = P::kTermBytes, kActBytes = P::kActBytes;
    constexpr int kOffAct = P::kOffAct, kOffW = P::kOffW, kOffAsf = P::kOffAsf, kOffWsf = P::kOffWsf;
    const Bars<kStages> bars{c.base + P::kOffBar};
    const uint32_t base = c.base;
    const unsigned long long tmo = c.tmo;
    uint32_t g = 0;
    bool ok = true;
    const UnitRing<kStages> ring{bars, c.units};
    grid_dep_wait();
    for (uint32_t i = 0; ok; ++i) {
        const int4 blk = ring.take(i, err_w, tmo, lane);
        if (blk.w < 0)
            break;
        const int ph = c.phase(blk.w), u = c.local(blk.w);
        const FcGemmArgs &a = *c.args[ph];
        const CUtensorMap *act_map = c.maps[ph][0], *act_map_sw = c.maps[ph][1], *act_map16 = c.maps[ph][2],
                          *w_map = c.maps[ph][3];
        const int kst = c.kst[ph], terms = c.terms[ph], scl_ld = a.K / 32;
        // the unit's fields the stage loop reads, in registers
        const bool fc1 = a.fc1 != 0, wsf_tiled = a.wsf_tiled != 0;
        const int R = a.R, act_rows = a.act_rows;
        const uint8_t *const wscale = a.wscale, *const act_sf = a.act_sf;
        const int nt0 = (u % c.n_groups[ph]) * kWT; // the unit's first weight tile
        const bool swap = !P::kWide && (kActRows < 128 || blk.z <= a.swap_rows); // wide: tokens on M always
        const int npad = (blk.z + 15) & ~15;
        const bool comb = swap && terms > 1 && npad <= P::kT2; // both terms on N of one MMA
        const int rb = blk.y / 128, o = blk.y & 127;
        // tokens on N: one box of kT2 rows per term plane covers the block (both terms, one copy),
        // else (blocks beyond kT2 rows) 16-row boxes per term, term 2 kTermBytes further on
        const bool sw3 = swap && npad <= P::kT2;
        const uint32_t act_bytes =
            (uint32_t)terms * (!swap ? (uint32_t)kTermBytes : sw3 ? (uint32_t)P::kT2 * 128u : (uint32_t)npad * 128u);
        // activation scales: one bulk copy of the two 128-row atoms (tokens on M); with the tokens
        // on N one bulk copy of the block's atom in the N layout where the producer of the
        // activations wrote one, else 4-byte copies of this block's rows into a stage atom laid
        // out for N; weight scales: one bulk copy (tiled layout) or 4-byte copies (row-major)
        const uint8_t *const act_sf_n =
            kScalesN && swap && a.act_sf_n && a.n_rows == P::kT2 && npad <= P::kT2 && (comb || terms == 1)
                ? a.act_sf_n + (size_t)(blk.y / P::kT2) * (size_t)kst * 512
                : nullptr;
        const uint32_t tx = act_bytes + kWT * kWTxBytes + (swap ? (act_sf_n ? 512u : 0u) : (uint32_t)terms * 512u) +
                            (a.wsf_tiled ? kWT * 512u : 0u);
        // tiled weight scales: the first tile's atoms, one per K stage, then the next tile's
        const uint8_t *wsf_tile = a.wscale + ((size_t)blk.x * a.n_tiles + nt0) * (size_t)kst * 512;
        // the second phase of a two-phase launch (FC2) reads h, which the first phase (FC1) writes:
        // it starts only once every FC1 unit of its row block has been counted
        if (ph == 1 && a.rb_done) {
            bool mine = true;
            if (elect_one())
                mine = wait_count(a.rb_done + u / c.n_groups[1], c.n_groups[0], err_w, tmo);
            if (!__all_sync(0xFFFFFFFFu, mine)) {
                ok = false;
                break;
            }
        }
        for (int kk = 0; kk < kst; ++kk, ++g) {
            if (P::producer_of(g) != PI)
                continue; // another producer warp fills this stage
            const int s = g % kStages;
            if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(bars.empty(s), ((g / kStages) & 1) ^ 1, err_w, tmo))) {
                ok = false;
                break;
            }
            // Every operand is computed by the whole (converged) warp; one elected lane issues the
            // stage's bulk copies (the weight tile first: it is the long pole, from DRAM), then the
            // whole warp issues the 4-byte scale copies, if any.
            const uint32_t full_s = bars.full(s);
            const uint32_t act = base + kOffAct + s * kActBytes;
            const uint32_t wdst = base + kOffW + s * P::kWStage;
            const uint32_t wsf = base + kOffWsf + s * P::kWsfStage;
            const uint32_t asf_dst = base + kOffAsf + s * kAsfBytes;
            const uint8_t *asf_src = act_sf + ((size_t)rb * kst + kk) * 1024;
            const int kx = kk * 128;
            if (elect_one()) {
                mbar_arrive_expect_tx(full_s, tx);
                // per weight tile nt: FC1 = gate rows [64 nt, 64 nt + 64) and the matching up rows, one
                // 3-D box; FC2 = rows [128 nt, 128 nt + 128), one box
                for (int wt = 0; wt < kWT; ++wt) {
                    const int nt = nt0 + wt;
                    if (fc1)
                        tma_load_3d(wdst + wt * kWBytes, w_map, kx, nt * 64, 2 * blk.x, full_s);
                    else
                        tma_load_2d(wdst + wt * kWBytes, w_map, kx, blk.x * R + nt * 128, full_s);
                    if (wsf_tiled)
                        bulk_copy_g2s(wsf + wt * kWsfBytes, wsf_tile + ((size_t)wt * kst + kk) * 512, 512u, full_s);
                }
                if (!swap) {
                    tma_load_3d(act, act_map, kx, blk.y, 0, full_s); // [terms][128 rows][128]
                    bulk_copy_g2s(asf_dst, asf_src, (uint32_t)terms * 512u, full_s);
                } else if (sw3) {
                    tma_load_3d(act, act_map_sw, kx, blk.y, 0, full_s); // [terms][kT2 rows][128]
                    if constexpr (kScalesN)
                        if (act_sf_n)
                            bulk_copy_g2s(asf_dst, act_sf_n + (size_t)kk * 512, 512u, full_s);
                } else {
                    for (int r16 = 0; r16 < npad; r16 += 16) {
                        tma_load_2d(act + r16 * 128, act_map16, kx, blk.y + r16, full_s);
                        if (terms > 1)
                            tma_load_2d(act + kTermBytes + r16 * 128, act_map16, kx, act_rows + blk.y + r16, full_s);
                    }
                }
            }
            __syncwarp();
            if (!wsf_tiled) // weight scale bytes: 4 per row (the stage's 4 blocks) into the atom layout
                for (int wt = 0; wt < kWT; ++wt) {
                    const int nt = nt0 + wt;
                    // tile rows as two 64-row halves: FC1 gate rows then the matching up rows
                    const int wrow_a = blk.x * R + (fc1 ? nt * 64 : nt * 128);
                    const int wrow_b = fc1 ? wrow_a + R / 2 : wrow_a + 64;
                    for (int r = lane; r < 128; r += 32) {
                        const int wr = r < 64 ? wrow_a + r : wrow_b + (r - 64);
                        cp_async_4(wsf + wt * kWsfBytes + sf_atom_offset(r, 0), wscale + (size_t)wr * scl_ld + kk * 4);
                    }
                }
            if (swap && !act_sf_n) {
                // row j of term t: from row o + j of the term's 128-row atom to N row t * kT2 + j of
                // one atom (both terms on N) or to row j of the term's own atom
                for (int j = lane; j < npad; j += 32)
                    for (int t = 0; t < terms; ++t)
                        cp_async_4(comb ? asf_dst + sf_atom_offset(t * P::kT2 + j, 0)
                                        : asf_dst + 512u * t + sf_atom_offset(j, 0),
                                   asf_src + 512 * t + sf_atom_offset(o + j, 0));
            }
            cp_async_mbar_arrive_noinc(full_s);
            __syncwarp();
        }
    }
    // drain: every stage this warp issued must have landed before the CTA may exit
    const uint32_t first = g > (uint32_t)kStages ? g - kStages : 0u;
    for (uint32_t q = first; q < g; ++q)
        if (P::producer_of(q) == PI)
            mbar_wait_bounded(bars.full(q % kStages), (q / kStages) & 1, nullptr, kDrainTimeoutNs);
}

// Scheduler role (one warp, one lane works): takes the CTA's work units from the launch's
// counter and publishes them kLook units ahead of the first reader, off the producers' path
// (the counter is a global atomic: a round trip of about a microsecond per unit).
template <int kActRows, int kMmaW, int kWTiles, int kTm>
__device__ __forceinline__ void scheduler_role(const Ctx &c, int lane)
{
    using P = Plan<kActRows, kMmaW, kWTiles, kTm>;
    const UnitRing<P::kStages> ring{Bars<P::kStages>{c.base + P::kOffBar}, c.units};
    if (lane == 0)
        for (uint32_t j = 0;
             ring.fill(j, *c.args[0], c.total_units, c.units0, c.n_groups[0], c.n_groups[1], c.tmo); ++j) {
        }
    __syncwarp();
}

// MMA role: warp 1 (MI = 0) and, with kMma = 2, warp 7 (MI = 1), taking stages g with
// g % kMma == MI.  The whole warp runs the loop, one elected lane issues.
template <int kActRows, int kMmaW, int kWTiles, int kTm, int MI>
__device__ __forceinline__ void mma_role(const Ctx &c)
{
    uint32_t *const err_w = c.err; // in a register: the stage loops wait with it
    using P = Plan<kActRows, kMmaW, kWTiles, kTm>;
    constexpr int kStages = P::kStages, kMma = P::kMma, kWT = P::kWT;
    constexpr int kTermBytes = P::kTermBytes, kActBytes = P::kActBytes;
    constexpr int kOffAct = P::kOffAct, kOffW = P::kOffW, kOffAsf = P::kOffAsf, kOffWsf = P::kOffWsf;
    const Bars<kStages> bars{c.base + P::kOffBar};
    const uint32_t base = c.base, tmem_base = c.tmem_base;
    const unsigned long long tmo = c.tmo;
    uint32_t g = 0, cnt = 0;
    bool ok = true;
    // this warp's scale-factor columns: the weight atoms at +0 (and +4 for a second tile), then
    // the activation atoms (one per term)
    const uint32_t sf_w = tmem_base + kSfCol + 16u * (uint32_t)MI;
    const uint32_t sf_act = sf_w + 4u * kWT;
    // descriptors of stage slot 0, K block 0 (term 1 of the activations, and the weights)
    const uint64_t dact0 = smem_desc_sw128(base + kOffAct), dw0 = smem_desc_sw128(base + kOffW);
    static_assert(P::kSmemBytes + 1024 < (1 << 18), "descriptor start field arithmetic needs addresses < 2^18");
    const UnitRing<kStages> ring{bars, c.units};
    const int lane = threadIdx.x & 31;
    for (; ok; ++cnt) {
        const int4 blk = ring.take(cnt, err_w, tmo, lane);
        if (blk.w < 0)
            break;
        const int phs = c.phase(blk.w); // the unit's phase (FC1 or FC2 in a two-phase launch)
        const FcGemmArgs &a = *c.args[phs];
        const int kst = c.kst[phs], terms = c.terms[phs];
        const bool swap = kActRows < 128 || blk.z <= a.swap_rows;
        const uint32_t npad = (uint32_t)((blk.z + 15) & ~15);
        const bool comb = swap && terms > 1 && npad <= (uint32_t)P::kT2;
        // MMAs per 32-element K block: one (both terms on N, or a single term) or one per term
        const bool t1 = !comb && terms > 1;
        const uint32_t idesc0 = swap ? idesc_mx(kFmtE2M1, kFmtE4M3, 128, comb ? P::kT2 + npad : npad, 0)
                                     : idesc_mx(kFmtE4M3, kFmtE2M1, 128, 128, 0);
        // scale columns of each MMA: tokens on N -> A = weight tile wt, B = activation term t;
        // tokens on M (one weight tile) -> A = activation term t, B = the weight tile
        uint32_t sfa[kWT][2], sfb[kWT][2];
#pragma unroll
        for (int wt = 0; wt < kWT; ++wt)
#pragma unroll
            for (int t = 0; t < 2; ++t) {
                sfa[wt][t] = swap ? sf_w + 4 * wt : sf_act + 4 * t;
                sfb[wt][t] = swap ? sf_act + 4 * t : sf_w + 4 * wt;
            }
        const int buf = cnt & 1;
        if (!__all_sync(0xFFFFFFFFu,
                        mbar_wait_bounded(bars.acc_empty(buf), ((cnt >> 1) & 1) ^ 1, err_w, tmo))) {
            ok = false;
            break;
        }
        tc_fence_after();
        // accumulator: one per buffer, or (64 columns apart) one per buffer and MMA warp or per
        // buffer and weight tile
        const uint32_t d = tmem_base + buf * 128 + (kMma > 1 ? 64u * (uint32_t)MI : 0u);
        bool first = true; // this warp's first stage of the unit initialises its accumulator
        for (int kk = 0; kk < kst; ++kk, ++g) {
            if (kMma > 1 && (int)(g % kMma) != MI)
                continue; // the other MMA warp takes this stage
            const int s = g % kStages;
            const uint32_t ph = (g / kStages) & 1;
            // The stage's operands are computed by the whole warp before the wait; then one elected
            // lane issues the scale copies, MMAs and commit back to back (measured: an elect /
            // reconverge around each instruction costs more than the instruction itself).
            const uint32_t wsf_s = base + kOffWsf + s * P::kWsfStage;
            const uint32_t asf_s = base + kOffAsf + s * kAsfBytes;
            // descriptors are affine in the address: the start field is address / 16 in the low
            // 14 bits, and every shared-memory address here stays below 2^18
            const uint64_t ds_act = dact0 + (uint64_t)((s * kActBytes) >> 4);
            const uint64_t ds_w = dw0 + (uint64_t)((s * P::kWStage) >> 4);
            uint64_t opa[4][kWT][2], opb[4][kWT][2];
            uint32_t idesc[4], accf[4];
#pragma unroll
            for (int k32 = 0; k32 < 4; ++k32) {
                // the scale-factor byte of this 32-element block sits in both sf-id fields
                idesc[k32] = idesc0 | ((uint32_t)k32 << 4) | ((uint32_t)k32 << 29);
                accf[k32] = (first && k32 == 0) ? 0u : 1u;
#pragma unroll
                for (int wt = 0; wt < kWT; ++wt) {
                    const uint64_t dw = ds_w + (uint64_t)((wt * kWBytes) >> 4) + 2u * k32; // +32 bytes per K block
#pragma unroll
                    for (int t = 0; t < 2; ++t) {
                        const uint64_t da = ds_act + (uint64_t)((t * kTermBytes) >> 4) + 2u * k32;
                        opa[k32][wt][t] = swap ? dw : da;
                        opb[k32][wt][t] = swap ? da : dw;
                    }
                }
            }
            const uint32_t empty_s = bars.empty(s);
            if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(bars.full(s), ph, err_w, tmo))) {
                ok = false;
                break;
            }
            tc_fence_after();
            if (elect_one()) {
                // scale atoms -> TMEM (in order with the MMAs below and with the previous stage's MMAs)
#pragma unroll
                for (int wt = 0; wt < kWT; ++wt)
                    tmem_cp_sf_atom(sf_w + 4 * wt, wsf_s + wt * kWsfBytes);
                tmem_cp_sf_atom(sf_act, asf_s);
                if (t1)
                    tmem_cp_sf_atom(sf_act + 4, asf_s + 512);
#pragma unroll
                for (int k32 = 0; k32 < 4; ++k32)
#pragma unroll
                    for (int wt = 0; wt < kWT; ++wt) {
                        umma_mx(d + (uint32_t)P::kAccW * wt, opa[k32][wt][0], opb[k32][wt][0], idesc[k32], sfa[wt][0],
                                sfb[wt][0],
                                accf[k32]);
                        if (t1)
                            umma_mx(d + (uint32_t)P::kAccW * wt, opa[k32][wt][1], opb[k32][wt][1], idesc[k32], sfa[wt][1],
                                    sfb[wt][1], 1u);
                    }
                umma_commit(empty_s);
            }
            __syncwarp();
            first = false;
        }
        if (ok && elect_one())
            umma_commit(bars.acc_full(buf));
        __syncwarp();
    }
    // all MMAs must have completed before TMEM is released
    if (elect_one())
        umma_commit(bars.mma_done());
    __syncwarp();
    mbar_wait_bounded(bars.mma_done(), 0, nullptr, kDrainTimeoutNs);
}

// MMA role of the wide variant (warp 1): per K block one M = 128 (token rows) x N = 256 (both
// weight tiles, contiguous in shared memory) block-scaled MMA per activation term, into the
// single accumulator at TMEM columns 0..255.  Scale factors: the two weight atoms at kSfCol and
// kSfCol + 4 (rows 0..127 and 128..255 of N), the activation atoms after them.
template <int kActRows, int kMmaW, int kWTiles, int kTm>
__device__ __forceinline__ void mma_role_wide(const Ctx &c)
{
    uint32_t *const err_w = c.err; // in a register: the stage loops wait with it
    using P = Plan<kActRows, kMmaW, kWTiles, kTm>;
    constexpr int kStages = P::kStages, kTermBytes = P::kTermBytes, kActBytes = P::kActBytes;
    const Bars<kStages> bars{c.base + P::kOffBar};
    const uint32_t base = c.base, tmem_base = c.tmem_base;
    const int kst = c.kst[0], terms = c.terms[0]; // one phase
    const unsigned long long tmo = c.tmo;
    uint32_t g = 0, cnt = 0;
    bool ok = true;
    const uint32_t sf_w = tmem_base + kSfCol, sf_act = sf_w + 8;
    const uint64_t dact0 = smem_desc_sw128(base + P::kOffAct), dw0 = smem_desc_sw128(base + P::kOffW);
    static_assert(P::kSmemBytes + 1024 < (1 << 18), "descriptor start field arithmetic needs addresses < 2^18");
    const uint32_t idesc0 = idesc_mx(kFmtE4M3, kFmtE2M1, 128, 256, 0);
    const UnitRing<kStages> ring{bars, c.units};
    const int lane = threadIdx.x & 31;
    for (; ok; ++cnt) {
        const int4 blk = ring.take(cnt, err_w, tmo, lane);
        if (blk.w < 0)
            break;
        // the accumulator is free once the epilogue has copied the previous unit's out of TMEM
        if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(bars.acc_empty(0), (cnt & 1) ^ 1, err_w, tmo))) {
            ok = false;
            break;
        }
        tc_fence_after();
        for (int kk = 0; kk < kst; ++kk, ++g) {
            const int s = g % kStages;
            const uint32_t ph = (g / kStages) & 1;
            const uint32_t wsf_s = base + P::kOffWsf + s * P::kWsfStage;
            const uint32_t asf_s = base + P::kOffAsf + s * kAsfBytes;
            const uint64_t ds_act = dact0 + (uint64_t)((s * kActBytes) >> 4);
            const uint64_t ds_w = dw0 + (uint64_t)((s * P::kWStage) >> 4);
            uint64_t opa[4][2], opb[4];
            uint32_t idesc[4], accf[4];
#pragma unroll
            for (int k32 = 0; k32 < 4; ++k32) {
                idesc[k32] = idesc0 | ((uint32_t)k32 << 4) | ((uint32_t)k32 << 29);
                accf[k32] = (kk == 0 && k32 == 0) ? 0u : 1u;
                opb[k32] = ds_w + 2u * k32; // +32 bytes per K block
#pragma unroll
                for (int t = 0; t < 2; ++t)
                    opa[k32][t] = ds_act + (uint64_t)((t * kTermBytes) >> 4) + 2u * k32;
            }
            const uint32_t empty_s = bars.empty(s);
            if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(bars.full(s), ph, err_w, tmo))) {
                ok = false;
                break;
            }
            tc_fence_after();
            if (elect_one()) {
                tmem_cp_sf_atom(sf_w, wsf_s);
                tmem_cp_sf_atom(sf_w + 4, wsf_s + kWsfBytes);
                tmem_cp_sf_atom(sf_act, asf_s);
                if (terms > 1)
                    tmem_cp_sf_atom(sf_act + 4, asf_s + 512);
#pragma unroll
                for (int k32 = 0; k32 < 4; ++k32) {
                    umma_mx(tmem_base, opa[k32][0], opb[k32], idesc[k32], sf_act, sf_w, accf[k32]);
                    if (terms > 1)
                        umma_mx(tmem_base, opa[k32][1], opb[k32], idesc[k32], sf_act + 4, sf_w, 1u);
                }
                umma_commit(empty_s);
            }
            __syncwarp();
        }
        if (ok && elect_one())
            umma_commit(bars.acc_full(0));
        __syncwarp();
    }
    // all MMAs must have completed before TMEM is released
    if (elect_one())
        umma_commit(bars.mma_done());
    __syncwarp();
    mbar_wait_bounded(bars.mma_done(), 0, nullptr, kDrainTimeoutNs);
}

// Epilogue of the wide variant: 8 warps, two per TMEM lane quarter; the warps of the first
// group (2..5) take weight tile 0 of the unit (accumulator columns 0..127), those of the second
// (kEpi2..kEpi2+3) tile 1 (columns 128..255).  A thread owns one token row: it copies its 128
// columns to registers, releases the accumulator, then forms its output (FC1: h = silu(gate) *
// up for the tile's 64 gate / 64 up rows, written as FC2's operand; FC2: f32 rows of Y).
template <int kActRows, int kMmaW, int kWTiles, int kTm>
__device__ __forceinline__ void epilogue_wide(const Ctx &c, int warp, int lane)
{
    uint32_t *const err_w = c.err; // in a register: the stage loops wait with it
    const FcGemmArgs &a = *c.args[0]; // one phase
    using P = Plan<kActRows, kMmaW, kWTiles, kTm>;
    const Bars<P::kStages> bars{c.base + P::kOffBar};
    const UnitRing<P::kStages> ring{bars, c.units};
    const int q = warp & 3;                     // TMEM lane quarter this warp may access
    const int half = warp >= P::kEpi2 ? 1 : 0;  // the unit's weight tile this warp writes
    for (uint32_t cnt = 0;; ++cnt) {
        const int4 blk = ring.take(cnt, err_w, c.tmo, lane);
        // the eight epilogue warps leave together (they share named barrier 2)
        if (!named_bar_all(2, 256, blk.w >= 0))
            break;
        const int nt = (blk.w % c.n_groups[0]) * 2 + half;
        const bool got = mbar_wait_bounded(bars.acc_full(0), cnt & 1, err_w, c.tmo);
        if (!named_bar_all(2, 256, got))
            break;
        tc_fence_after();
        const uint32_t tb = c.tmem_base + ((uint32_t)(32 * q) << 16) + 128u * half;
        uint32_t v[8][16];
#pragma unroll
        for (int j = 0; j < 8; ++j)
            tmem_ld16(tb + 16 * j, v[j]);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(bars.acc_empty(0)); // the MMA warp may overwrite the accumulator now
        if (a.fc1) {
            const int rl = 32 * q + lane;
            const bool valid = rl < blk.z;
            const int row = blk.y + rl;
            // columns 0..63: gate rows nt*64 + i, columns 64..127: the matching up rows.  Both halves'
            // h first, so that the accumulator registers are dead before the encoder runs.
            float h[2][32];
#pragma unroll
            for (int c32 = 0; c32 < 2; ++c32)
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    h[c32][i] = silu_mul(__uint_as_float(v[2 * c32][i]), __uint_as_float(v[4 + 2 * c32][i]));
                    h[c32][16 + i] = silu_mul(__uint_as_float(v[2 * c32 + 1][i]), __uint_as_float(v[5 + 2 * c32][i]));
                }
            if (valid) {
#pragma unroll
                for (int c32 = 0; c32 < 2; ++c32)
                    store_act_block32(a.hq, a.hsf, a.hq_rows, a.out_ld, row, nt * 64 + 32 * c32, h[c32], a.act_mxfp8);
            }
        } else {
            // FC2: f32 rows of Y.  Stored straight from registers, each store instruction of the
            // warp would write 32 rows' 16-byte pieces (half sectors, 32 segments).  Instead each
            // 16-column chunk goes through this warp's 2 KB buffer ([32 rows][4 x 16 bytes]) and
            // comes back out as 8 rows x 64 contiguous bytes per instruction: whole sectors.  Row
            // r's 16-byte piece i sits at position i ^ ((r >> 1) & 3): a 16-byte access serves 8
            // lanes per shared-memory wavefront, and the 8 lanes of either side (rows l .. l + 7
            // writing piece i; rows r, r + 1 reading pieces 0..3) then meet 8 distinct bank groups.
            uint4 *stg = reinterpret_cast<uint4 *>(c.ystage + 2048 * (half * 4 + (warp & 3)));
            const int r0 = lane >> 2, ch = lane & 3;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    stg[lane * 4 + (i ^ ((lane >> 1) & 3))] =
                        make_uint4(v[j][4 * i], v[j][4 * i + 1], v[j][4 * i + 2], v[j][4 * i + 3]);
                __syncwarp();
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    const int r = 8 * p + r0; // row of this warp's 32
                    const uint4 val = stg[r * 4 + (ch ^ ((r >> 1) & 3))];
                    if (32 * q + r < blk.z)
                        *reinterpret_cast<uint4 *>(a.y + (size_t)(blk.y + 32 * q + r) * a.out_ld + nt * 128 + 16 * j +
                                                   4 * ch) = val;
                }
                __syncwarp();
            }
        }
    }
}

// kScalesN: the activation scales of units with their tokens on N may come in the N layout (one
// bulk copy per stage), and FC1 writes h's scales in that layout too; a separate instantiation, so
// that the kernels without it keep their code as it was (measured: carrying both forms in one
// kernel slowed FC1 at 256 tokens by 2-8 %, and even a dead argument in its epilogue by 2 %).
template <int kActRows, int kMmaW, int kWTiles, int kTm, bool kTwo, bool kScalesN>
__global__ void __launch_bounds__(Plan<kActRows, kMmaW, kWTiles, kTm>::kThreads, 1)
    fc_gemm_kernel(const __grid_constant__ FcGemmArgs a0, const __grid_constant__ FcGemmArgs a1,
                   const __grid_constant__ CUtensorMap act_map, const __grid_constant__ CUtensorMap act_map_sw,
                   const __grid_constant__ CUtensorMap act_map16, const __grid_constant__ CUtensorMap w_map,
                   const __grid_constant__ CUtensorMap act_map1, const __grid_constant__ CUtensorMap act_map_sw1,
                   const __grid_constant__ CUtensorMap act_map16_1, const __grid_constant__ CUtensorMap w_map1)
{
    using P = Plan<kActRows, kMmaW, kWTiles, kTm>;
    constexpr int kStages = P::kStages;
    constexpr int kOffX = P::kOffX, kOffBar = P::kOffBar, kOffTmemSlot = P::kOffTmemSlot;
    constexpr int kProd = P::kProd, kMma = P::kMma;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *const gsm = smem_raw + (base - raw);
    const Bars<kStages> bars{base + kOffBar};
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // warp roles: 0 producer 0, 1 MMA 0 (+ TMEM owner), 2..5 epilogue, 6 producer 1, 7 MMA 1

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(bars.full(s), 1 + 32);  // producer's expect_tx + 32 cp.async arrivals
            mbar_init(bars.empty(s), 1);      // the commit of the MMA warp that took the stage
        }
        mbar_init(bars.mma_done(), kMma);
        for (int b = 0; b < 2; ++b) {
            mbar_init(bars.acc_full(b), kMma); // every MMA warp commits every unit
            mbar_init(bars.acc_empty(b), 32 * P::kEpiWarps);
        }
        for (int r = 0; r < kRing; ++r) {
            mbar_init(bars.ring_full(r), 1);                             // the scheduler's publish
            mbar_init(bars.ring_empty(r), kProd + kMma + P::kEpiWarps);  // one release per reading warp
        }
        fence_mbar_init();
        fence_proxy_async_smem();
        prefetch_tensormap(&act_map);
        prefetch_tensormap(&act_map_sw);
        prefetch_tensormap(&act_map16);
        prefetch_tensormap(&w_map);
        if (kTwo) { // two phases: FC2's maps too
            prefetch_tensormap(&act_map1);
            prefetch_tensormap(&act_map_sw1);
            prefetch_tensormap(&act_map16_1);
            prefetch_tensormap(&w_map1);
        }
    }
    if (warp == 1) {
        tmem_alloc(base + kOffTmemSlot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t *>(gsm + kOffTmemSlot);
    // The next kernel may launch now: what it reads of this kernel's output it reads after its
    // own grid_dep_wait; what it reads before (the row-block list, the work-unit counters) was
    // written two kernels back, which had completed before this kernel could launch.
    if (threadIdx.x == 0)
        grid_dep_launch();

    // one phase (a0 alone), or two (kTwo: a0 = FC1, a1 = FC2)
    constexpr bool two = kTwo;
    const int nrb = *a0.num_rowblocks;
    const unsigned long long tmo = a0.timeout_ns;
    Ctx ctx;
    ctx.base = base;
    ctx.units = reinterpret_cast<volatile int *>(gsm + P::kOffUnits);
    ctx.ystage = gsm + P::kOffY;
    ctx.tmem_base = tmem_base;
    ctx.args[0] = &a0;
    ctx.args[1] = two ? &a1 : &a0;
    ctx.maps[0][0] = &act_map;
    ctx.maps[0][1] = &act_map_sw;
    ctx.maps[0][2] = &act_map16;
    ctx.maps[0][3] = &w_map;
    ctx.maps[1][0] = two ? &act_map1 : &act_map;
    ctx.maps[1][1] = two ? &act_map_sw1 : &act_map_sw;
    ctx.maps[1][2] = two ? &act_map16_1 : &act_map16;
    ctx.maps[1][3] = two ? &w_map1 : &w_map;
    for (int ph = 0; ph < 2; ++ph) {
        const FcGemmArgs &ap = *ctx.args[ph];
        ctx.n_groups[ph] = ap.n_tiles / P::kWT;       // the launch guarantees n_tiles % kWT == 0
        ctx.kst[ph] = ap.K / 128;                     // K stages of 128 elements (4 scale blocks)
        ctx.terms[ph] = kTm == 1 ? 1 : ap.terms;      // activation terms per row: 1 (w4a8) or 2 (w4a16)
    }
    ctx.units0 = nrb * ctx.n_groups[0];
    ctx.total_units = ctx.units0 + (two ? nrb * ctx.n_groups[1] : 0);
    ctx.tmo = tmo;
    ctx.err = a0.err;
    ctx.two = kTwo;
    if (warp == 0) {
        producer_role<kActRows, kMmaW, kWTiles, kTm, 0, kScalesN>(ctx, lane);
    } else if (warp >= 6 && warp < 5 + kProd) {
        // further producer warps (compile-time role index: every TMA operand stays warp-uniform)
        if (warp == 6)
            producer_role<kActRows, kMmaW, kWTiles, kTm, 1 % kProd, kScalesN>(ctx, lane);
        else if (warp == 7)
            producer_role<kActRows, kMmaW, kWTiles, kTm, 2 % kProd, kScalesN>(ctx, lane);
        else if (warp == 8)
            producer_role<kActRows, kMmaW, kWTiles, kTm, 3 % kProd, kScalesN>(ctx, lane);
    } else if (warp == 1) {
        if constexpr (P::kWide)
            mma_role_wide<kActRows, kMmaW, kWTiles, kTm>(ctx);
        else
            mma_role<kActRows, kMmaW, kWTiles, kTm, 0>(ctx);
    } else if (P::kWide && ((warp >= 2 && warp < 6) || (warp >= P::kEpi2 && warp < P::kEpi2 + 4))) {
        epilogue_wide<kActRows, kMmaW, kWTiles, kTm>(ctx, warp, lane);
    } else if (kMma > 1 && warp == 5 + kProd) {
        mma_role<kActRows, kMmaW, kWTiles, kTm, (kMma > 1 ? 1 : 0)>(ctx);
    } else if (warp == P::kThreads / 32 - 1) {
        scheduler_role<kActRows, kMmaW, kWTiles, kTm>(ctx, lane);
    } else if (warp >= 2 && warp < 6) {
        // ------------------------------------------------------------ epilogue (warps 2..5)
        const int q = warp & 3; // TMEM lane quarter this warp may access
        uint32_t *const err_w = a0.err;
        float *xch = reinterpret_cast<float *>(gsm + kOffX);
        const UnitRing<kStages> ring{bars, reinterpret_cast<volatile int *>(gsm + P::kOffUnits)};
        uint32_t g_run = 0; // pipeline stages of the units before this one
        for (uint32_t cnt = 0;; ++cnt) {
            const int4 blk = ring.take(cnt, err_w, tmo, lane);
            // the four epilogue warps leave together (they share named barriers below)
            if (!named_bar_all(2, 128, blk.w >= 0))
                break;
            const int phs = ctx.phase(blk.w), u = ctx.local(blk.w);
            const FcGemmArgs &a = *ctx.args[phs];
            const int kst = ctx.kst[phs], terms = ctx.terms[phs];
            const uint32_t g0 = g_run; // the unit's first stage
            g_run += (uint32_t)kst;
            const int nt0 = (u % ctx.n_groups[phs]) * P::kWT; // the unit's first weight tile
            const int rows = blk.z;
            const bool swap = kActRows < 128 || rows <= a.swap_rows;
            const int buf = cnt & 1;
            // the four epilogue warps leave together or not at all (they share named barrier 1 below)
            const bool got = mbar_wait_bounded(bars.acc_full(buf), (cnt >> 1) & 1, err_w, tmo);
            if (!named_bar_all(2, 128, got))
                break;
            tc_fence_after();
            const uint32_t tb = tmem_base + ((uint32_t)(32 * q) << 16) + buf * 128;
            if (!swap) {
                // thread = one grouped row; TMEM columns = the tile's 128 weight rows (one tile)
                const int nt = nt0;
                const int rl = 32 * q + lane;
                const bool valid = rl < rows;
                const int row = blk.y + rl;
                if (a.fc1) {
                    // columns 0..63 gate, 64..127 up, for i = nt*64 + c
                    for (int c32 = 0; c32 < 2; ++c32) {
                        uint32_t g0[16], g1[16], u0[16], u1[16];
                        tmem_ld16(tb + 32 * c32, g0);
                        tmem_ld16(tb + 32 * c32 + 16, g1);
                        tmem_ld16(tb + 64 + 32 * c32, u0);
                        tmem_ld16(tb + 64 + 32 * c32 + 16, u1);
                        tmem_wait_ld();
                        float h[32];
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            h[i] = silu_mul(__uint_as_float(g0[i]), __uint_as_float(u0[i]));
                            h[16 + i] = silu_mul(__uint_as_float(g1[i]), __uint_as_float(u1[i]));
                        }
                        if (valid)
                            store_act_block32(a.hq, a.hsf, a.hq_rows, a.out_ld, row, nt * 64 + 32 * c32, h,
                                              a.act_mxfp8);
                    }
                } else {
                    float *orow = a.y + (size_t)row * a.out_ld + nt * 128;
                    for (int c = 0; c < 8; ++c) {
                        uint32_t y0[16];
                        tmem_ld16(tb + 16 * c, y0);
                        tmem_wait_ld();
                        if (valid) {
                            uint4 *dst = reinterpret_cast<uint4 *>(orow + 16 * c);
#pragma unroll
                            for (int i = 0; i < 4; ++i)
                                dst[i] = make_uint4(y0[4 * i], y0[4 * i + 1], y0[4 * i + 2], y0[4 * i + 3]);
                        }
                    }
                }
            } else {
                // lane L of the tile = weight row; TMEM columns = tokens
                const int L = 32 * q + lane;
                const int npad = (rows + 15) & ~15;
                const bool comb = terms > 1 && npad <= P::kT2;
                // partial sums: per MMA warp with stages in this unit (with one K stage only the
                // warp that took it), and per term when both terms sit side by side on N
                const bool acc0 = kMma == 1 || kst > 1 || (g0 & 1) == 0;
                const bool acc1 = kMma > 1 && (kst > 1 || (g0 & 1) == 1);
                for (int wt = 0; wt < P::kWT; ++wt) // each weight tile of the unit (64 columns apart)
                for (int n0 = 0; n0 < npad; n0 += 16) {
                    const int nt = nt0 + wt;
                    float v[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        v[j] = 0.f;
                    for (int w = 0; w < kMma; ++w) {
                        if (!(w == 0 ? acc0 : acc1))
                            continue;
                        for (int t = 0; t < (comb ? 2 : 1); ++t) {
                            uint32_t r[16];
                            tmem_ld16(tb + 64 * w + P::kAccW * wt + (t ? P::kT2 : 0) + n0, r);
                            tmem_wait_ld();
#pragma unroll
                            for (int j = 0; j < 16; ++j)
                                v[j] += __uint_as_float(r[j]);
                        }
                    }
                    if (a.fc1) {
                        // the up rows live in lanes 64..127: hand them to the gate lanes through smem
                        if (q >= 2) {
#pragma unroll
                            for (int j = 0; j < 16; ++j)
                                xch[(L - 64) * 16 + j] = v[j];
                        }
                        named_bar_sync(1, 128);
                        if (q < 2) {
                            const int i = nt * 64 + L;
                            for (int j = 0; j < 16; ++j) {
                                const int n = n0 + j;
                                if (n >= rows)
                                    break;
                                const float hv = silu_mul(v[j], xch[L * 16 + j]);
                                if constexpr (kScalesN)
                                    store_act_warp32(a.hq, a.hsf, a.hq_rows, a.out_ld, blk.y + n, i, hv,
                                                     a.act_mxfp8, lane, a.hsf_n, a.n_rows);
                                else
                                    store_act_warp32(a.hq, a.hsf, a.hq_rows, a.out_ld, blk.y + n, i, hv,
                                                     a.act_mxfp8, lane);
                            }
                        }
                        named_bar_sync(1, 128);
                    } else {
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const int n = n0 + j;
                            if (n < rows)
                                a.y[(size_t)(blk.y + n) * a.out_ld + nt * 128 + L] = v[j];
                        }
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(bars.acc_empty(buf));
            if (a.fc1 && a.rb_done) {
                // two phases: count this FC1 unit done for its row block once every epilogue thread's h
                // stores are visible device-wide (FC2's producers wait for the count, then copy h)
                __threadfence();
                named_bar_sync(1, 128);
                if (q == 0 && lane == 0) {
                    __threadfence();
                    atomicAdd(a.rb_done + u / ctx.n_groups[0], 1);
                }
            }
            if (swap && !a.fc1 && a.fuse_combine)
                fused_combine_unit(a, blk, nt0, P::kWT, 32 * q + lane, reinterpret_cast<int *>(xch));
        }
    }

    tc_fence_before();
    // every CTA waits for the kernel before it at least once, also a CTA that got no work (only
    // the producers wait otherwise), so that this grid completes only after its predecessor has
    if (threadIdx.x == 0)
        grid_dep_wait();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

template <int kActRows, int kMmaW, int kWTiles, int kTm, bool kTwo = false, bool kScalesN = false>
static cudaError_t prepare_one()
{
    return cudaFuncSetAttribute(fc_gemm_kernel<kActRows, kMmaW, kWTiles, kTm, kTwo, kScalesN>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                Plan<kActRows, kMmaW, kWTiles, kTm>::kSmemBytes);
}

cudaError_t fc_gemm_prepare()
{
    cudaError_t e;
    if ((e = prepare_one<16, 1, 1, 2>()) != cudaSuccess || (e = prepare_one<16, 2, 1, 2>()) != cudaSuccess ||
        (e = prepare_one<16, 1, 2, 2>()) != cudaSuccess || (e = prepare_one<16, 1, 4, 2>()) != cudaSuccess ||
        (e = prepare_one<32, 1, 1, 2>()) != cudaSuccess ||
        (e = prepare_one<32, 2, 1, 2>()) != cudaSuccess || (e = prepare_one<32, 1, 2, 2>()) != cudaSuccess ||
        (e = prepare_one<64, 1, 1, 2>()) != cudaSuccess || (e = prepare_one<128, 1, 1, 2>()) != cudaSuccess ||
        (e = prepare_one<128, 1, 1, 1>()) != cudaSuccess || (e = prepare_one<128, 1, 2, 2>()) != cudaSuccess)
        return e;
    if ((e = prepare_one<128, 1, 2, 1>()) != cudaSuccess || (e = prepare_one<16, 2, 1, 2, true>()) != cudaSuccess)
        return e;
    if ((e = prepare_one<16, 2, 1, 2, false, true>()) != cudaSuccess ||
        (e = prepare_one<16, 1, 2, 2, false, true>()) != cudaSuccess ||
        (e = prepare_one<16, 1, 4, 2, false, true>()) != cudaSuccess)
        return e;
    return prepare_one<16, 2, 1, 2, true, true>();
}

template <int kActRows, int kMmaW, int kWTiles, int kTm, bool kScalesN = false>
static void launch_one(const FcGemmArgs &a, const CUtensorMap &act_map, const CUtensorMap &act_map_sw,
                       const CUtensorMap &act_map16, const CUtensorMap &w_map, int grid, cudaStream_t s, bool pdl)
{
    using P = Plan<kActRows, kMmaW, kWTiles, kTm>;
    launch_kernel(fc_gemm_kernel<kActRows, kMmaW, kWTiles, kTm, false, kScalesN>, dim3(grid), dim3(P::kThreads),
                  (size_t)P::kSmemBytes, s, pdl, a, a, act_map, act_map_sw, act_map16, w_map, act_map, act_map_sw,
                  act_map16, w_map);
}

void launch_fc_gemm(const FcGemmArgs &a, const CUtensorMap &act_map, const CUtensorMap &act_map_sw,
                    const CUtensorMap &act_map16, const CUtensorMap &w_map, int grid, cudaStream_t s, bool pdl)
{
    // Row blocks of at most 16 / 32 / 64 rows run with their tokens on N; smaller activation
    // tiles leave room for more pipeline stages (bytes in flight) in the weight-streaming shapes.
    // Small batches (tokens on N): FC1 with two MMA warps on alternate stages; FC2 (short
    // units) with one MMA warp and two weight tiles per work unit when the tiles pair up.
    // Each choice measured fastest on the decode shapes.
    const bool wt2 = !a.fc1 && a.n_tiles % 2 == 0;
    // the N-layout scales (a.act_sf_n, a.hsf_n) are read and written by the kScalesN
    // instantiations only; the others ignore them
    const bool sn = a.act_sf_n != nullptr || a.hsf_n != nullptr;
    if (a.max_block_rows <= 16) {
        if (a.fc1 && sn)
            launch_one<16, 2, 1, 2, true>(a, act_map, act_map_sw, act_map16, w_map, grid, s, pdl);
        else if (a.fc1)
            launch_one<16, 2, 1, 2>(a, act_map, act_map_sw, act_map16, w_map, grid, s, pdl);
        else if (a.fc2_tiles == 4 && a.n_tiles % 4 == 0 && sn)
            launch_one<16, 1, 4, 2, true>(a, act_map, act_map_sw, act_map16, w_map, grid, s, pdl);
        else if (a.fc2_tiles == 4 && a.n_tiles % 4 == 0)
            launch_one<16, 1, 4, 2>(a, act_map, act_map_sw, act_map16, w_map, grid, s, pdl);
        else if (wt2 && sn)
            launch_one<16, 1, 2, 2, true>(a, act_map, act_map_sw, act_map16, w_map, grid, s, pdl);
        else if (wt2)
            launch_one<16, 1, 2, 2>(a, act_map, act_map_sw, act_map16, w_map, grid, s, pdl);
        else
            launch_one<16, 1, 1, 2>(a, act_map, act_map_sw, act_map16, w_map, grid, s, pdl);
    } else if (a.max_block_rows <= 32) {
        if (a.fc1)
            launch_one<32, 2, 1, 2>(a, act_map, act_map_sw, act_map16, w_map, grid, s, pdl);
        else if (wt2)
            launch_one<32, 1, 2, 2>(a, act_map, act_map_sw, act_map16, w_map, grid, s, pdl);
        else
            launch_one<32, 1, 1, 2>(a, act_map, act_map_sw, act_map16, w_map, grid, s, pdl);
    } else if (a.max_block_rows <= 64) {
        launch_one<64, 1, 1, 2>(a, act_map, act_map_sw, act_map16, w_map, grid, s, pdl);
    } else if (a.wide && a.n_tiles % 2 == 0) {
        // the wide variant (two weight tiles per unit, N = 256 MMAs): half the activation bytes
        // per MMA of the one-tile variant (the 128-row GEMMs were bound by the shared-memory fill
        // from L2, not by the tensor pipe)
        if (a.terms == 1)
            launch_one<128, 1, 2, 1>(a, act_map, act_map_sw, act_map16, w_map, grid, s, pdl);
        else
            launch_one<128, 1, 2, 2>(a, act_map, act_map_sw, act_map16, w_map, grid, s, pdl);
    } else if (a.terms == 1) {
        // single-term activations (w4a8 FC1): the smaller stages leave room for 6 of them
        // instead of 4, i.e. more bytes in flight per SM
        launch_one<128, 1, 1, 1>(a, act_map, act_map_sw, act_map16, w_map, grid, s, pdl);
    } else {
        launch_one<128, 1, 1, 2>(a, act_map, act_map_sw, act_map16, w_map, grid, s, pdl);
    }
}

void launch_fc_gemm_two_phase(const FcGemmArgs &a1, const CUtensorMap *maps1, const FcGemmArgs &a2,
                              const CUtensorMap *maps2, int grid, cudaStream_t s, bool pdl)
{
    // tokens on N, 16-row blocks, two MMA warps: the small-batch FC1 variant serves both phases
    // (FC2 units then take one weight tile each)
    using P = Plan<16, 2, 1, 2>;
    if (a1.act_sf_n != nullptr || a1.hsf_n != nullptr)
        launch_kernel(fc_gemm_kernel<16, 2, 1, 2, true, true>, dim3(grid), dim3(P::kThreads), (size_t)P::kSmemBytes, s,
                      pdl, a1, a2, maps1[0], maps1[1], maps1[2], maps1[3], maps2[0], maps2[1], maps2[2], maps2[3]);
    else
        launch_kernel(fc_gemm_kernel<16, 2, 1, 2, true, false>, dim3(grid), dim3(P::kThreads), (size_t)P::kSmemBytes,
                      s, pdl, a1, a2, maps1[0], maps1[1], maps1[2], maps1[3], maps2[0], maps2[1], maps2[2], maps2[3]);
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
