// Channel-skipping decode attention on the tensor cores: INT2 codes, four
// query heads per KV head (the GQA 4:1 shape of the Dual-QK workloads), and
// the whole decode step -- append, channel choice, attention -- fused into one
// launch on the same page machinery.
//
// "Dual-QK: Sharp Queries and Flat Keys for Prunable 2-bit KV Caches":
//   §3.1 keys enter the cache transformed (K' = K A), queries are transformed
//        by A^{-T}, so transformed scores equal the original ones;
//   §3.2 Eq. 4: one channel mask per KV head from the pooled query energy;
//        scores over the retained channels only, 1/sqrt(d) with the full d;
//   §3.3 only the key rows selected by the mask are read from each 128-token
//        page; values and metadata are read in full;
//   §3.4 one softmax over every token (online per warp, merged per CTA and
//        then across CTAs), followed by value aggregation.
//
// Both contractions of a page are small dense GEMMs once the codes are
// unpacked, and they run as mma.sync m16n8k16 (f16 in, f32 accumulate):
//   scores^T[token][head] = codes^T[token][channel] . q'[channel][head]
//   out^T[channel][head]  = codes[channel][token]   . w[token][head]
// Codes stay exact: a 2-bit field masked in place inside a 16-bit half is an
// fp16 subnormal equal to code * 2^(pos-24), so unpacking is one AND per two
// codes; the power of two is compensated exactly on the other operand or in
// fp32 afterwards.  The query is split into fp16 hi + lo parts, which occupy
// the two columns of each head in the score MMAs (n = 8 = 4 heads x {hi,lo}):
// scores need near-fp32 operands because the softmax exponentiates them.  The
// score k-steps run over all 128 channel rows of a page with q' = 0 on the
// channels that are not selected, so every k-step lies inside one key group
// and its per-token scale is applied in fp32 afterwards.  Softmax weights
// enter the value MMAs as fp16 (the usual flash-attention rounding of P; the
// error it adds is below 6e-4 of the output's largest entry); value MMAs take
// a group pair per tile (rows: 8 channels of each group, columns: 4 heads x 2
// groups) so the per-token value scale is folded into the weights once per
// group.  The value zero-point term sum_t p(t) z(t) is one more MMA.
//
// Work split: one CTA = one (sequence, KV head, split), eight warps in four
// pairs.  A pair processes one 128-token page at a time from a two-stage ring
// filled by bulk asynchronous copies completing on an mbarrier: key rows are
// copied in 64-byte chunks (two rows, the unit in which the memory system
// fetches anyway) as a few runs of chunks that hold a selected row, into their
// own place in the stage, and the tail of the page (value codes, channel 0,
// metadata) in one copy.  Warp w of the pair takes half w of every 16-token
// word of the page (64 tokens) and keeps its own online softmax; its softmax
// weights pass from the score layout to the value layout through a small
// buffer of its own.
//
// Page schedule (without RoPE buckets): the pages a unit reads form a pool,
// taken from the last page backwards and dealt round-robin to the unit's
// pairs.  The schedule is fixed by the shapes alone, so results are
// reproducible bit for bit.  The tail of a page (everything but the key rows)
// does not depend on the channel choice, so a pair copies the tails of its
// first two pages, and brings their key rows into L2, before the choice is
// loaded.  With RoPE buckets each split reads a contiguous range of pages,
// one segment per bucket.
//
// The fused step kernel (kvq_decode_step without RoPE buckets) runs as
// clusters of two CTAs, the two taking consecutive splits of one (sequence,
// KV head).  CTA r of a cluster computes q' for channels 64r..64r+63 (64
// columns of A^{-T}, staged in shared memory around the first pages' tails;
// the same fixed-order float64 arithmetic as kvq_select_channels, the four
// heads' chains side by side in one thread) and their pooled energies; after a
// cluster barrier both CTAs read the 128 energies and all of q' through
// distributed shared memory and make the same channel choice.  The first
// cluster holds the pages of the new tokens (the first pool pages): its CTA r
// transforms, quantizes and writes key groups 2r and 2r+1 of them (the
// arithmetic of kvq_append; code bits are OR-ed into positions that are still
// zero) before the same barrier, so those pages are staged after it.  (Pairs
// of CTAs pack the SMs' two CTA slots exactly; clusters of four leave slots of
// some GPCs unused.)
//
// With RoPE buckets a step is two launches: the preparation kernel
// (kvq_select.cu: the channel choice of every bucket, the page plans and the
// append of the step's new tokens) and this decode as its programmatic
// dependent.  The decode's CTAs start while the preparation runs and stream
// the tails of pages that hold no new token; they wait for it only before
// they read what it writes (the plans, the new tokens' pages and protected
// slots), then copy their plan in with 16-byte loads.
#include "kvq_internal.cuh"

#include <cooperative_groups.h>

namespace kvq {
namespace {

constexpr int kPairs = 4;
constexpr int kThreads = 64 * kPairs;
constexpr int kWarps = kThreads / 32;
static_assert(kWarps == 8, "one warp per score k-step in the plan");
constexpr int kKeyBytes = 128 * 32;               // key code rows of a page
constexpr int kFixBytes = fixed_bytes(2);         // value codes, ch0, metadata (groups of 32)
constexpr int kStageBytes = kKeyBytes + kFixBytes;
static_assert(kStageBytes == page_bytes(2) && page_bytes(2, 1) <= kStageBytes, "a stage holds one page image");
constexpr int kChunks = kKeyBytes / 64;           // 64-byte chunks of key rows
static_assert(kChunks == kPlanChunks, "the plan's chunks are the page's");
constexpr uint32_t kWaitPolls = 1u << 20;         // bound on mbarrier polls per stage
constexpr int kStepMaxNew = 4;                    // new tokens per fused step
constexpr int kCluster = 2;                       // CTAs per cluster of the fused step
constexpr int kCols = kD / kCluster;              // channels whose q' one CTA of a cluster computes
constexpr int kAppendRounds = 2;                  // rounds the appending cluster's pairs sit out

struct __align__(16) MmaShared {
    uint8_t stage[kPairs][2][kStageBytes];
    uint64_t mbar[kPairs][2];
    uint4 pex[kWarps][4][8];           // per warp: fp16 softmax weights [head][8-token block]
    PagePlan plan;                     // score-MMA operands and copy list of the channel choice
    float q[4][kD];                    // qsel of the 4 heads, by selected position
    int chan_pos[kD];                  // channel -> position in the selected list, -1 = not selected
    uint32_t touched[2];               // chunk bitmask halves
    uint32_t selmask[4];               // fused step: the channel choice, 128 bits
    int s_len;
    double qp_own[4][kCols];           // fused step: q' of this CTA's channels (read by the cluster)
    double e2_own[kCols];              // and their pooled energies
    double trange[kWarps][4];          // fused step, one grid per token: per-warp key / value ranges
};
// Prologue scratch of the fused step.  Before the page loop the staging
// memory P holds the 64-column block of A^{-T} as 128 rows of 512 bytes.  A
// CTA that appends nothing keeps the tails of its pairs' first pages in
// flight into stage 0 meanwhile, so its rows go around them: rows 32p..32p+7
// in the key area of pair p's stage 0, rows 32p+8..32p+31 in its stage 1.  A
// CTA that appends (the first cluster, the tier cluster) holds the block in
// P[0, 64K); A's column block then follows it through P[0, 96K) in two
// halves (below), and no stage is in flight during the prologue.
// Energies, ranks and the gathered q' come after the q' chains in the same
// memory (outside the first tails).
constexpr int kBlkRowBytes = kCols * (int)sizeof(double);        // 512
constexpr int kOffAHi = 0;                                        // A rows 64..127
constexpr int kOffALo = kD * kBlkRowBytes;                        // A rows 0..63
constexpr int kOffE2 = kOffALo + 64 * kBlkRowBytes;               // double[128]
constexpr int kOffRank = kOffE2 + kD * (int)sizeof(double);       // int[2][128]
constexpr int kOffQp = kStageBytes;                               // double[4][128] in stage[0][1], after the append
static_assert(kOffRank + 2 * kD * (int)sizeof(int) <= kPairs * 2 * kStageBytes, "scratch fits the stages");
static_assert(kOffQp + 4 * kD * (int)sizeof(double) <= 2 * kStageBytes, "q' copy inside stage[0][1]");
static_assert(kOffE2 >= 3 * 2 * kStageBytes + kStageBytes && kOffQp >= kStageBytes,
              "energies, ranks and q' lie outside the stage-0 tails of the first pages");
static_assert(8 * kBlkRowBytes <= kKeyBytes && 24 * kBlkRowBytes <= kStageBytes,
              "32 rows of the A^{-T} block per pair around its first tail");
struct PexScratch {                    // in MmaShared::pex
    double qin[kD][4];                 // query rows, float64 (exact for bf16 / f32 inputs), [channel][head]
};
// new key rows: float (exact) in MmaShared::q until the channel choice, then
// float64 in the staging memory freed by the A^{-T} block; new value rows in
// registers, then float64 after the key rows.  With a value rotation its
// 64-column block follows A's through the same two halves of the staging
// memory (rows 0..63 where A's were, then rows 64..127).
constexpr int kOffKs = kBlkRowBytes * 64;                         // past the high rows of A
constexpr int kOffVs = kOffKs + kStepMaxNew * kD * (int)sizeof(double);
static_assert(kOffVs + kStepMaxNew * kD * (int)sizeof(double) <= kOffALo, "new rows below the low rows of A");
constexpr int kVPre = kStepMaxNew * kD / kThreads;                 // value elements per thread
static_assert(kVPre * kThreads == kStepMaxNew * kD, "value rows split evenly over the threads");
static_assert(sizeof(PexScratch) <= sizeof(((MmaShared *)0)->pex), "query and key rows fit the exchange buffers");


__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// the same with a zero accumulator in
__device__ __forceinline__ void mma16816_z(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                           uint32_t a3, uint32_t b0, uint32_t b1) {
    const float z = 0.f;
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%10,%10,%10,%10};\n"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(z));
}

// barrier of the two warps of a pair that also ANDs a flag over them
__device__ __forceinline__ bool pair_sync_and(int pair, bool v) {
    uint32_t r;
    asm volatile(
        "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.and.pred q, %2, 64, p;\n selp.u32 %0, 1, 0, q;\n}\n"
        : "=r"(r) : "r"((uint32_t)v), "r"(pair + 1) : "memory");
    return r != 0;
}

// After a give-up: wait (bounded by kWaitPolls) until the stage's copies
// have landed, so that no copy still writes into shared memory when the CTA
// goes on to reuse it or exits.
__device__ __forceinline__ void drain_stage(uint32_t bar, uint32_t parity) {
    for (uint32_t i = 0; i < kWaitPolls; i++)
        if (mbar_try_wait(bar, parity)) return;
}

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint32_t h2u(__half2 h) { return *reinterpret_cast<uint32_t *>(&h); }
__device__ __forceinline__ __half2 u2h(uint32_t u) { return *reinterpret_cast<__half2 *>(&u); }
__device__ __forceinline__ float lo_f16(uint32_t w) { return __half2float(__ushort_as_half((uint16_t)(w & 0xffffu))); }
__device__ __forceinline__ float hi_f16(uint32_t w) { return __half2float(__ushort_as_half((uint16_t)(w >> 16))); }

// 4-token metadata chunk c of group g (the page format's XOR permutation)
__device__ __forceinline__ int meta_chunk(int g, int c) { return c ^ (((c >> 3) & 3) ^ ((g & 1) << 2)); }

// context split of this CTA: pages [blk0, blk1) of the first `len` tokens
struct Split {
    int blk0, blk1;
};
__device__ __forceinline__ Split split_of(int len, int S, int s) {
    const int nblk = (len + kT - 1) / kT;
    const int bps = (nblk + S - 1) / S;
    const int blk0 = s * bps;
    return {blk0, min(nblk, blk0 + bps)};
}

// The page schedule of a unit without RoPE buckets.  The pages that hold the
// coded tokens [lo, hi) are [P0, P1); pool index q is page P1 - 1 - q (the
// last page first: it holds a step's new tokens).  The unit's NP = kPairs *
// S_pages pairs take the pool round-robin, pair P = kPairs s + pair taking
// q = P in round 0.  With `skip` > 0 the first `appenders` pairs (the fused
// step's appending cluster) sit out rounds 1..skip, which the other pairs
// take in turn, so the work of appending makes no straggler.  The schedule is
// a pure function of the shapes: every run assigns the same pages to the
// same pairs in the same order, so results are reproducible bit for bit.
struct Pool {
    int P0, P1;
    int P, NP;                 // this pair's index and the pairs of the unit
    int appenders, skip;
    int pre;                   // the tails of this pair's first `pre` pages are already in flight
    __device__ int size() const { return P1 - P0; }
    __device__ int page(int q) const { return P1 - 1 - q; }
    // pool index of this pair's j-th page, -1 past the end
    __device__ int index(int j) const {
        const int A = appenders, K = skip;
        int q;
        if (j == 0)
            q = P;
        else if (P < A)
            q = NP + K * (NP - A) + (j - 1) * NP + P;
        else if (j <= K)
            q = NP + (j - 1) * (NP - A) + (P - A);
        else
            q = NP + K * (NP - A) + (j - K - 1) * NP + P;
        return q < size() ? q : -1;
    }
};
__device__ __forceinline__ Pool unit_pool(int lo, int hi, int s, int pair, int S_pages) {
    Pool p;
    p.P0 = lo / kT;
    p.P1 = hi > lo ? (hi + kT - 1) / kT : p.P0;
    p.P = kPairs * s + pair;
    p.NP = kPairs * S_pages;
    p.appenders = 0;
    p.skip = 0;
    p.pre = 0;
    return p;
}
// The page plan from the channel choice (sh.chan_pos, sh.q, and the
// zero-point sums already in sh.plan.qg): score-MMA B fragments, channel 0's
// q' and the copy list of a page.  Called by every thread after a barrier
// that follows the last write of chan_pos / q; ends with a barrier.
template <int NG>
__device__ __forceinline__ void build_plan(MmaShared &sh, int tid, int warp, int lane) {
    // B fragments of k-step `warp`: channel 0 and unselected channels get q' = 0
    auto qf = [&](int hh, int c) -> float {
        const int p = sh.chan_pos[c];
        return p >= 1 ? sh.q[hh][p] : 0.f;
    };
    sh.plan.bq[warp][lane] = make_uint2(plan_bq_word(warp, lane, 0, qf), plan_bq_word(warp, lane, 1, qf));
    if (tid < 4) sh.plan.q0[tid] = sh.q[tid][0];
    // 64-byte chunks of key rows that hold a selected row
    if (tid < kChunks) {
        const bool t = sh.chan_pos[2 * tid] >= 1 || sh.chan_pos[2 * tid + 1] >= 1;
        const unsigned m = __ballot_sync(0xffffffffu, t);
        if (lane == 0) sh.touched[warp] = m;
    }
    __syncthreads();
    if (warp == 0) plan_copies_warp(sh.plan, (uint64_t)sh.touched[0] | ((uint64_t)sh.touched[1] << 32), NG, lane);
    __syncthreads();
}

// Copies of one page into stage st of a pair, issued by one thread: the tail
// (value codes, channel 0, metadata) expects its bytes without arriving; the
// key chunks arrive on the barrier, so the stage's phase completes once both
// parts have landed.
template <int NG>
__device__ __forceinline__ void issue_tail(MmaShared &sh, int pair, int st, const uint8_t *src) {
    constexpr uint32_t kFix = (uint32_t)fixed_bytes(2, NG);
    const uint32_t bar = smem_u32(&sh.mbar[pair][st]);
    mbar_expect_tx(bar, kFix);
    bulk_g2s(smem_u32(sh.stage[pair][st]) + kKeyBytes, src + kKeyBytes, kFix, bar);
}
__device__ __forceinline__ void issue_keys(MmaShared &sh, int pair, int st, const uint8_t *src) {
    const uint32_t bar = smem_u32(&sh.mbar[pair][st]);
    const uint32_t dst = smem_u32(sh.stage[pair][st]);
    mbar_arrive_expect_tx(bar, sh.plan.tx_keys);
    const int n = sh.plan.n_copies - 1;
    for (int r = 0; r < n; r++) {
        const uint2 c = sh.plan.copy[r];
        bulk_g2s(dst + c.x, src + c.x, c.y, bar);
    }
}

// The page loop and the merges.  Tokens outside [lo, hi) (beyond the length,
// or in the protected tier) are left out of the softmax.
//  DYN (no RoPE buckets): this pair's pages of the unit's round-robin
//    schedule `pool`, each staged while the one before it is computed.
//    The tails of its first pool.pre (0..2) pages are already in flight
//    into stages 0 and 1.
//  static: pages [sp.blk0, sp.blk1), pair `pair` taking every kPairs-th.
//    With RoPE buckets of w_pages pages the split runs as segments, one per
//    bucket: before each, every warp is done with the previous one and
//    load_seg(bucket) puts that bucket's channel choice and page plan in place
//    (called by every thread; it ends with a barrier); the softmax state runs
//    on across segments.  w_pages = 0: one segment, the plan already in place.
// A wait that gives up (mbar_wait_bounded) stops the pair on both of its warps
// (the flag is ANDed over the pair at its barrier): no further copy is issued,
// the stage still in flight is drained after the loop, and the call's result
// is reported invalid through KVQ_DEV_TIMEOUT.
template <int NG, bool DYN, typename SegFn>
__device__ __forceinline__ void run_pages(MmaShared &sh, const uint8_t *__restrict__ unit_pages, int lo, int hi,
                                          Split sp, const Pool &pool, int S, int s, size_t qrow0,
                                          float *__restrict__ part_o, float2 *__restrict__ part_ml,
                                          float *__restrict__ out, uint32_t *counter, uint32_t *status,
                                          uint32_t polls, const double *rot, int w_pages, SegFn &&load_seg) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int pair = warp >> 1, half = warp & 1;
    const int gid = lane >> 2, tig = lane & 3;
    const int hh = gid >> 1, part = gid & 1;

    // Channel-0 coefficient of head tig, and the B fragment of the score
    // zero-point MMA: k-slot 2tig holds group tig's sum of kept q' of head
    // gid >> 1 (hi or lo fp16 part by gid & 1), every other k-slot 0; both
    // pre-scaled to the base-2 score domain (reloaded for each bucket's
    // segment)
    float q0_t = 0.f;
    uint32_t bz = 0;
    auto load_coef = [&]() {
        q0_t = sh.plan.q0[tig] * kScoreScaleLog2;
        bz = tig < NG ? (uint32_t)f16_part(sh.plan.qg[hh][tig] * kScoreScaleLog2, part) : 0u;
    };
    load_coef();

    float m_run = -INFINITY;      // running max of head tig (base-2 domain)
    float l_thr = 0.f;            // this thread's share of the running sum of head tig
    float co[8][4];               // out^T tiles; [0]: channel a, head tig; [3]: channel b, head tig
    float cz[4];                  // value zero-point term: [0] = group gid, head tig
#pragma unroll
    for (int mt = 0; mt < 8; mt++)
#pragma unroll
        for (int r = 0; r < 4; r++) co[mt][r] = 0.f;
#pragma unroll
    for (int r = 0; r < 4; r++) cz[r] = 0.f;

    const uint32_t half_sel = half ? 0x7632u : 0x5410u;      // this warp's 16-bit half of a word
    const uint32_t vx_sel = half ? 0x4332u : 0x4110u;        // {half, high byte of half}
    const float zmask = gid < NG ? 1.f : 0.f;                // z-term rows: one per group
    uint4 *pexw = &sh.pex[warp][0][0];

    // one page `pg` staged in `cur`: scores, online softmax, value aggregation
    auto page = [&](const uint8_t *cur, int pg) {
        const uint8_t *vcodes = cur + kKeyBytes;
        const uint32_t *ch0w = reinterpret_cast<const uint32_t *>(vcodes + 128 * 32);
        const uint32_t *kmeta = reinterpret_cast<const uint32_t *>(vcodes + 128 * 32 + 256);
        const uint32_t *vmeta = kmeta + NG * kT;

        // ---------------- scores: tokens 16gid + 8half + 2i + r, head tig
        float sc[4][2];
#pragma unroll
        for (int i = 0; i < 4; i++) sc[i][0] = sc[i][1] = 0.f;
        const uint8_t *kb = cur + tig * 32 + 4 * gid;
#pragma unroll
        for (int g = 0; g < NG; g++) {
            constexpr int KS = 8 / NG;                  // k-steps (16 channels each) per key group
            float C[4][4];
#pragma unroll
            for (int j = 0; j < KS; j++) {
                const int ks = KS * g + j;
                const uint8_t *sb = kb + ks * 512;
                const uint32_t Wa = *reinterpret_cast<const uint32_t *>(sb);
                const uint32_t Wb = *reinterpret_cast<const uint32_t *>(sb + 4 * 32);
                const uint32_t Wc = *reinterpret_cast<const uint32_t *>(sb + 8 * 32);
                const uint32_t Wd = *reinterpret_cast<const uint32_t *>(sb + 12 * 32);
                const uint32_t Xab = __byte_perm(Wa, Wb, half_sel), Xcd = __byte_perm(Wc, Wd, half_sel);
                const uint32_t Yab = Xab >> 8, Ycd = Xcd >> 8;
                const uint2 bb = sh.plan.bq[ks][lane];
#pragma unroll
                for (int i = 0; i < 4; i++) {
                    const uint32_t x1 = (i & 2) ? Yab : Xab;
                    const uint32_t x2 = (i & 2) ? Ycd : Xcd;
                    const uint32_t m0 = 0x00030003u << (4 * (i & 1));
                    const uint32_t m1 = m0 << 2;
                    if (j == 0)
                        mma16816_z(C[i], x1 & m0, x1 & m1, x2 & m0, x2 & m1, bb.x, bb.y);
                    else
                        mma16816(C[i], x1 & m0, x1 & m1, x2 & m0, x2 & m1, bb.x, bb.y);
                }
            }
            // scale of group g for the thread's 8 tokens
#pragma unroll
            for (int q4 = 0; q4 < 2; q4++) {
                const uint4 w = *reinterpret_cast<const uint4 *>(
                    kmeta + 128 * g + 4 * meta_chunk(g, 4 * gid + 2 * half + q4));
                const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int e = 0; e < 4; e++) {
                    const int tt = 4 * q4 + e, i = tt >> 1, r = tt & 1;
                    sc[i][r] = fmaf(lo_f16(ws[e]), C[i][2 * r] + C[i][2 * r + 1], sc[i][r]);
                }
            }
        }
        // zero-point term sum_g zero_g(t) qgsum_g, one MMA per tile: thread
        // tig puts its group's fp16 zero point (exact) of tokens T and T+1
        // (rows gid and gid+8) into k-slot 2tig; the rest of A is 0
        float Cz[4][4];
        {
            const int zg = tig < NG ? tig : 0;
            uint32_t zw[8];
#pragma unroll
            for (int q4 = 0; q4 < 2; q4++) {
                const uint4 w = *reinterpret_cast<const uint4 *>(
                    kmeta + 128 * zg + 4 * meta_chunk(zg, 4 * gid + 2 * half + q4));
                zw[4 * q4] = w.x; zw[4 * q4 + 1] = w.y; zw[4 * q4 + 2] = w.z; zw[4 * q4 + 3] = w.w;
            }
            const uint32_t zkeep = tig < NG ? 0xffffffffu : 0u;
#pragma unroll
            for (int i = 0; i < 4; i++)
                mma16816_z(Cz[i], (zw[2 * i] >> 16) & zkeep, (zw[2 * i + 1] >> 16) & zkeep, 0u, 0u, bz, 0u);
        }
        // full scores (base-2 domain), masked beyond the sequence on the last page
        float mx = -INFINITY;
        {
            const uint4 w = *reinterpret_cast<const uint4 *>(ch0w + 8 * gid + 4 * half);
            const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int i = 0; i < 4; i++) {
#pragma unroll
                for (int r = 0; r < 2; r++) {
                    const float c0v = __uint_as_float(r ? (ws[i] & 0xffff0000u) : (ws[i] << 16));
                    // 2^(24 - field position) undoes the code scaling; times log2(e)/sqrt(d)
                    const float comp = __int_as_float((127 + 24 - 4 * (i & 1) - 2 * r) << 23) * kScoreScaleLog2;
                    sc[i][r] = fmaf(sc[i][r], comp, fmaf(q0_t, c0v, Cz[i][2 * r] + Cz[i][2 * r + 1]));
                }
            }
            if (pg * kT < lo || (pg + 1) * kT > hi) {       // page with tokens outside [lo, hi)
                const int tok0 = pg * kT + 16 * gid + 8 * half;
#pragma unroll
                for (int i = 0; i < 4; i++)
#pragma unroll
                    for (int r = 0; r < 2; r++) {
                        const int tok = tok0 + 2 * i + r;
                        if (tok < lo || tok >= hi) sc[i][r] = -INFINITY;
                    }
            }
#pragma unroll
            for (int i = 0; i < 4; i++) mx = fmaxf(mx, fmaxf(sc[i][0], sc[i][1]));
        }
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
        const float m_new = fmaxf(m_run, mx);
        // a half-page with no valid token leaves this warp's state unchanged
        const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
        const float alpha = ex2(m_run - m_use);
        float psum = 0.f;
#pragma unroll
        for (int i = 0; i < 4; i++)
#pragma unroll
            for (int r = 0; r < 2; r++) {
                sc[i][r] = ex2(sc[i][r] - m_use);
                psum += sc[i][r];
            }
        m_run = m_new;
        l_thr = fmaf(l_thr, alpha, psum);
        if (!__all_sync(0xffffffffu, alpha == 1.f)) {
#pragma unroll
            for (int mt = 0; mt < 8; mt++) {
                co[mt][0] *= alpha;
                co[mt][3] *= alpha;
            }
            cz[0] *= alpha;
        }

        // ---------------- softmax weights: score layout -> value layout.
        // Local token l = 8 * block + e; the value MMAs take tokens (f, f+4)
        // of a block as one fp16 pair, scaled by 4^(3-f) to offset the code
        // scale of field f; word f of (head, block) holds that pair.
        {
            uint32_t wv[4];
#pragma unroll
            for (int f = 0; f < 4; f++) {
                const float F = (float)(1 << (2 * (3 - f)));
                const int i0 = f >> 1, r0 = f & 1;           // token f = 2 i0 + r0, token f+4 = 2(i0+2) + r0
                wv[f] = h2u(__floats2half2_rn(sc[i0][r0] * F, sc[i0 + 2][r0] * F));
            }
            pexw[tig * 8 + gid] = make_uint4(wv[0], wv[1], wv[2], wv[3]);
        }
        __syncwarp();
        // value k-step j = 2u + v uses fields f0 = 2v (k-slots 2tig, 2tig+1) and
        // f1 = 2v+1 (k-slots 2tig+8, 2tig+9) of word 2tig+u's half, i.e. local
        // tokens (f, f+4) of block 2tig+u
        uint32_t ph[4][2];
#pragma unroll
        for (int u = 0; u < 2; u++) {
            const uint4 w = pexw[hh * 8 + 2 * tig + u];
            ph[2 * u][0] = w.x;
            ph[2 * u][1] = w.y;
            ph[2 * u + 1][0] = w.z;
            ph[2 * u + 1][1] = w.w;
        }

        // ---------------- values: tile mt = group pair pp, rows 8 channels of
        // each group; this thread's weight column belongs to group 2pp + part
#pragma unroll
        for (int pp = 0; pp < 2; pp++) {
            const int gv = NG == 1 ? 0 : 2 * pp + part;
            uint32_t bw[4][2];
            {
                uint32_t vw[2][8];             // {s, z} of local tokens 8(2tig+u) + e, group gv
#pragma unroll
                for (int u = 0; u < 2; u++)
#pragma unroll
                    for (int c = 0; c < 2; c++) {
                        const uint4 w = *reinterpret_cast<const uint4 *>(
                            vmeta + 128 * gv + 4 * meta_chunk(gv, 4 * (2 * tig + u) + 2 * half + c));
                        vw[u][4 * c] = w.x; vw[u][4 * c + 1] = w.y; vw[u][4 * c + 2] = w.z; vw[u][4 * c + 3] = w.w;
                    }
#pragma unroll
                for (int j = 0; j < 4; j++) {
                    const int u = j >> 1;
#pragma unroll
                    for (int r = 0; r < 2; r++) {
                        const int f = 2 * (j & 1) + r;
                        const __half2 sp2 = u2h(__byte_perm(vw[u][f], vw[u][f + 4], 0x5410));
                        bw[j][r] = h2u(__hmul2(u2h(ph[j][r]), sp2));
                    }
                }
            }
#pragma unroll
            for (int sub = 0; sub < 4; sub++) {
                const int mt = 4 * pp + sub;
                const int ca = 64 * pp + 8 * sub + gid;
                const uint2 r0 = *reinterpret_cast<const uint2 *>(vcodes + ca * 32 + 8 * tig);
                const uint2 r1 = *reinterpret_cast<const uint2 *>(vcodes + (ca + 32) * 32 + 8 * tig);
                const uint32_t x0[2] = {__byte_perm(r0.x, 0u, vx_sel), __byte_perm(r0.y, 0u, vx_sel)};
                const uint32_t x1[2] = {__byte_perm(r1.x, 0u, vx_sel), __byte_perm(r1.y, 0u, vx_sel)};
#pragma unroll
                for (int j = 0; j < 4; j++) {
                    const int u = j >> 1;
                    const uint32_t mA = 0x00030003u << (4 * (j & 1));
                    const uint32_t mB = mA << 2;
                    mma16816(co[mt], x0[u] & mA, x1[u] & mA, x0[u] & mB, x1[u] & mB, bw[j][0], bw[j][1]);
                }
            }
        }
        // zero-point term: rows = groups (row gid holds group gid), times p
        {
            uint32_t zw[2][8];
            const int zg = NG == 1 ? 0 : (gid & 3);
#pragma unroll
            for (int u = 0; u < 2; u++)
#pragma unroll
                for (int c = 0; c < 2; c++) {
                    const uint4 w = *reinterpret_cast<const uint4 *>(
                        vmeta + 128 * zg + 4 * meta_chunk(zg, 4 * (2 * tig + u) + 2 * half + c));
                    zw[u][4 * c] = w.x; zw[u][4 * c + 1] = w.y; zw[u][4 * c + 2] = w.z; zw[u][4 * c + 3] = w.w;
                }
#pragma unroll
            for (int j = 0; j < 4; j++) {
                const int u = j >> 1;
                uint32_t a[2];
#pragma unroll
                for (int r = 0; r < 2; r++) {
                    const int f = 2 * (j & 1) + r;
                    const __half2 sc2 = __float2half2_rn(zmask / (float)(1 << (2 * (3 - f))));
                    a[r] = h2u(__hmul2(u2h(__byte_perm(zw[u][f], zw[u][f + 4], 0x7632)), sc2));
                }
                mma16816(cz, a[0], 0u, a[1], 0u, ph[j][0], ph[j][1]);
            }
        }
    };

    const bool issuer = (tid & 63) == 0;
    // after a give-up: the stage still in flight (bit 0) and its parity (bit
    // 1), bit 2: stage 1's first phase too (a tail copied ahead); -1: none
    int pend = -1;
    if constexpr (DYN) {
        // this pair's pages of the schedule, the next one staged while the
        // current one is computed; the same sequence on both warps
        int q_cur = pool.index(0);
        if (issuer && q_cur >= 0) {
            const uint8_t *src = unit_pages + (size_t)pool.page(q_cur) * page_bytes(2, NG);
            if (pool.pre < 1) issue_tail<NG>(sh, pair, 0, src);
            issue_keys(sh, pair, 0, src);
        }
        for (int it = 0; q_cur >= 0; it++) {
            const int st = it & 1;
            const uint32_t par = (uint32_t)(it >> 1) & 1u;
            bool ok = mbar_wait_bounded(smem_u32(&sh.mbar[pair][st]), par, status, polls);
            ok = pair_sync_and(pair, ok);                        // both warps left the other stage
            if (!ok) {
                pend = st | (int)(par << 1);
                if (it == 0 && pool.pre >= 2) {
                    // the second page's tail is in flight without its key
                    // copies: complete that phase's arrival so it can drain
                    if (issuer) mbar_arrive(smem_u32(&sh.mbar[pair][1]));
                    pend |= 4;
                }
                break;
            }
            const int q_next = pool.index(it + 1);
            if (issuer && q_next >= 0) {
                const uint8_t *src = unit_pages + (size_t)pool.page(q_next) * page_bytes(2, NG);
                if (it + 1 >= pool.pre) issue_tail<NG>(sh, pair, st ^ 1, src);
                issue_keys(sh, pair, st ^ 1, src);
            }
            page(sh.stage[pair][st], pool.page(q_cur));
            q_cur = q_next;
        }
    } else {
        int it = 0;                   // pages this pair has staged (the ring position, across segments)
        bool dead = false;            // a wait gave up: no more copies, no more pages
        for (int seg0 = sp.blk0; seg0 < sp.blk1;) {
            const int seg1 = w_pages > 0 ? min(sp.blk1, (seg0 / w_pages + 1) * w_pages) : sp.blk1;
            if (w_pages > 0) {
                __syncthreads();                                 // every warp is done with the last plan
                load_seg(seg0 / w_pages);
                load_coef();
            }
            const int first = seg0 + pair;
            if (issuer && !dead && first < seg1) {
                const uint8_t *src = unit_pages + (size_t)first * page_bytes(2, NG);
                issue_tail<NG>(sh, pair, it & 1, src);
                issue_keys(sh, pair, it & 1, src);
            }
            for (int pg = first; pg < seg1 && !dead; pg += kPairs, it++) {
                const int st = it & 1;
                const uint32_t par = (uint32_t)(it >> 1) & 1u;
                bool ok = mbar_wait_bounded(smem_u32(&sh.mbar[pair][st]), par, status, polls);
                ok = pair_sync_and(pair, ok);                    // both warps left the other stage
                if (!ok) {
                    dead = true;
                    pend = st | (int)(par << 1);
                    break;
                }
                if (issuer && pg + kPairs < seg1) {
                    const uint8_t *src = unit_pages + (size_t)(pg + kPairs) * page_bytes(2, NG);
                    issue_tail<NG>(sh, pair, st ^ 1, src);
                    issue_keys(sh, pair, st ^ 1, src);
                }
                page(sh.stage[pair][st], pg);
            }
            seg0 = seg1;
        }
    }
    // a stage whose wait gave up may still receive bytes: wait (bounded)
    // until they have landed before the staging memory is reused below
    if (pend >= 0) {
        drain_stage(smem_u32(&sh.mbar[pair][pend & 1]), (uint32_t)(pend >> 1) & 1u);
        if (pend & 4) drain_stage(smem_u32(&sh.mbar[pair][1]), 0u);
    }

    // ------------------------------------------------------------ merge
    // per warp: head tig's max, sum and output; then across the 8 warps
    float l_head = l_thr;
    l_head += __shfl_xor_sync(0xffffffffu, l_head, 4);
    l_head += __shfl_xor_sync(0xffffffffu, l_head, 8);
    l_head += __shfl_xor_sync(0xffffffffu, l_head, 16);
    float zsum[NG];
#pragma unroll
    for (int g = 0; g < NG; g++) zsum[g] = __shfl_sync(0xffffffffu, cz[0], 4 * g + tig);
    __syncthreads();                                     // stages are free now
    float *mo = reinterpret_cast<float *>(sh.stage[0][0]);       // [warp][head][128]
    float *mml = mo + kWarps * 4 * kD;                           // [warp][head][2]
    constexpr float kCodeScale = 262144.f;                       // 2^18
#pragma unroll
    for (int mt = 0; mt < 8; mt++) {
        const int pp = mt >> 2, ca = 64 * pp + 8 * (mt & 3) + gid;
        mo[(warp * 4 + tig) * kD + ca] = fmaf(co[mt][0], kCodeScale, zsum[NG == 1 ? 0 : 2 * pp]);
        mo[(warp * 4 + tig) * kD + ca + 32] = fmaf(co[mt][3], kCodeScale, zsum[NG == 1 ? 0 : 2 * pp + 1]);
    }
    if (gid == 0) {
        mml[(warp * 4 + tig) * 2] = m_run;
        mml[(warp * 4 + tig) * 2 + 1] = l_head;
    }
    __syncthreads();
    for (int e = tid; e < 4 * kD; e += kThreads) {
        const int hl = e / kD, c = e % kD;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kWarps; w++) M = fmaxf(M, mml[(w * 4 + hl) * 2]);
        float o = 0.f, L = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < kWarps; w++) {
                const float wt = exp2f(mml[(w * 4 + hl) * 2] - M);
                L = fmaf(wt, mml[(w * 4 + hl) * 2 + 1], L);
                o = fmaf(wt, mo[(w * 4 + hl) * kD + c], o);
            }
        }
        const size_t row = (qrow0 + hl) * S + s;
        part_o[row * kD + c] = o;
        if (c == 0) part_ml[row] = make_float2(M, L);
    }
    static_assert(merge_scratch_floats(4, kThreads, 256) * 4 <= 2 * 2 * kStageBytes, "merge scratch fits stages 2-3");
    merge_unit_if_last<4, kThreads>(part_o, part_ml, S, qrow0, out, counter,
                                    reinterpret_cast<float *>(sh.stage[2][0]), rot);
}

// A CTA that handles the protected tier instead of pages: half `half_idx` of
// the unit's slots, then the split merge.  The query coefficients and channel
// lists come from `qs` (a TierQShared or TierQBuckets).
template <typename QS>
__device__ __forceinline__ void tier_cta_q(MmaShared &sh, const uint8_t *slots, int len, int n_sink, int n_recent,
                                           int half_idx, int k, const QS &qs, float *part_o, float2 *part_ml,
                                           size_t qrow0, int S, int s, float *out, uint32_t *counter,
                                           const double *rot) {
    float *scratch = reinterpret_cast<float *>(sh.stage[0][0] + kD * sizeof(int));
    static_assert(kD * sizeof(int) + tier_scratch_floats(4) * 4 <= 2 * (size_t)kStageBytes * 2,
                  "tier scratch ends before the merge scratch in stages 2-3");
    const int NP = n_sink + n_recent, per = (NP + 1) / 2;
    const int slot0 = min(NP, half_idx * per), slot1 = min(NP, slot0 + per);
    tier_partial<4, kThreads>(slots, len, n_sink, n_recent, slot0, slot1, qs, k, part_o, part_ml, qrow0, S, s,
                              scratch);
    merge_unit_if_last<4, kThreads>(part_o, part_ml, S, qrow0, out, counter, reinterpret_cast<float *>(sh.stage[2][0]),
                                    rot);
}
// The same with the one channel choice in sh.chan_pos / sh.q (a barrier after
// their last write).
__device__ __forceinline__ void tier_cta(MmaShared &sh, const uint8_t *slots, int len, int n_sink, int n_recent,
                                         int half_idx, int k, float *part_o, float2 *part_ml, size_t qrow0, int S,
                                         int s, float *out, uint32_t *counter, const double *rot) {
    int *list = reinterpret_cast<int *>(sh.stage[0][0]);                    // position -> channel
    const int tid = threadIdx.x;
    if (tid < kD) list[tid] = 0;
    __syncthreads();
    if (tid < kD && sh.chan_pos[tid] >= 0) list[sh.chan_pos[tid]] = tid;
    __syncthreads();
    tier_cta_q(sh, slots, len, n_sink, n_recent, half_idx, k, TierQShared{&sh.q[0][0], kD, 1, list}, part_o,
               part_ml, qrow0, S, s, out, counter, rot);
}

// ---------------------------------------------------------------- decode
// With RoPE buckets (BK; w_pages > 0 pages each, nbk entries per selection
// array) each split reads a contiguous range of pages and, per bucket its
// pages fall in, that bucket's channel choice; the tier CTAs read each
// protected position's own bucket's.  Without buckets the pages come from the
// unit's round-robin schedule, and the tails of each pair's first two pages
// are in flight, and their key rows on their way to L2, while the channel
// choice is loaded.
//
// STEP: the second launch of a decode step, a programmatic dependent of the
// preparation kernel (the channel choices, page plans and the append of the
// step's n_new tokens, kvq_select.cu).  Until griddepcontrol.wait it reads
// only what that kernel does not write -- the length before the step and the
// tails of pages that hold no new token -- and it advances the length after
// the wait, once every CTA of the sequence has read it.  Its page plans come
// from `plans` ([unit][bucket]); the three-call decode builds them from the
// channel lists.
template <int NG, bool BK, bool STEP>
__global__ void __launch_bounds__(kThreads, 2)
decode_mma_kernel(const uint8_t *__restrict__ pages, int32_t *__restrict__ seq_len, int Hkv,
                  int NB, int Hq, const int32_t *__restrict__ idx, const float *__restrict__ qsel,
                  const float *__restrict__ qgsum, int k, float *__restrict__ part_o,
                  float2 *__restrict__ part_ml, int S, float *__restrict__ out,
                  uint32_t *__restrict__ counters, uint32_t *__restrict__ status,
                  int n_sink, int n_recent, const double *__restrict__ v_rot, int nbk, int w_pages,
                  uint32_t polls, int n_new, const PagePlan *__restrict__ plans) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    MmaShared &sh = *reinterpret_cast<MmaShared *>(smem_raw);

    const int s = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const double *rot = v_rot ? v_rot + (size_t)h * kD * kD : nullptr;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const size_t unit = (size_t)b * Hkv + h;
    const size_t qrow0 = (size_t)b * Hq + (size_t)h * 4;

    // channel choice of bucket bk into shared memory, then the page plan.
    // The list must be channel 0 followed by ascending channels in 1..127;
    // any other list reads no key rows and raises KVQ_DEV_INDEX.
    auto load_sel = [&](int bk) {
        for (int e = tid; e < 4 * k; e += kThreads) {
            const int hl = e / k, i = e % k;
            sh.q[hl][i] = qsel[((qrow0 + hl) * nbk + bk) * k + i];
        }
        if (tid < 4 * kNG)
            sh.plan.qg[tid / kNG][tid % kNG] = qgsum[((qrow0 + tid / kNG) * nbk + bk) * kNG + tid % kNG];
        if (tid < kD) sh.chan_pos[tid] = -1;
        const int32_t *sel = idx + (unit * nbk + bk) * k;
        int my_c = -1;
        bool bad = false;
        if (tid < k) {
            my_c = sel[tid];
            bad = (tid == 0) ? my_c != 0 : (my_c <= sel[tid - 1] || my_c > kD - 1);
        }
        const bool any_bad = __syncthreads_or(bad);
        if (any_bad && tid == 0) atomicOr(status, (uint32_t)KVQ_DEV_INDEX);
        if (!any_bad && tid < k) sh.chan_pos[my_c] = tid;
        __syncthreads();
        build_plan<NG>(sh, tid, warp, lane);
    };
    // the preparation kernel's plan of bucket bk (after the wait)
    auto load_plan = [&](int bk) {
        const uint4 *src = reinterpret_cast<const uint4 *>(plans + unit * nbk + bk);
        uint4 *dst = reinterpret_cast<uint4 *>(&sh.plan);
        for (int e = tid; e < (int)(sizeof(PagePlan) / 16); e += kThreads) dst[e] = __ldcg(src + e);
        __syncthreads();
    };

    if (tid < 2 * kPairs) mbar_init(smem_u32(&sh.mbar[tid >> 1][tid & 1]), 1);
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    // the length (with the step's new tokens once they are in; a step that
    // would overflow the capacity appends nothing)
    const int L0 = seq_len[b];
    const bool fits = L0 >= 0 && L0 + n_new <= NB * kT;
    const int len = min(max(STEP && fits ? L0 + n_new : L0, 0), NB * kT);
    __syncthreads();                              // barriers initialised before copies complete on them
    // after the preparation kernel: wait for it, make its page writes visible
    // to the bulk copies, and advance the length once every CTA of sequence b
    // has read it (its completion counter reaches S * Hkv)
    auto after_prep = [&]() {
        if constexpr (STEP) {
            asm volatile("griddepcontrol.wait;\n" ::: "memory");
            asm volatile("fence.proxy.async.global;\n" ::: "memory");
            if (tid == 0) {
                const unsigned prev = atomicAdd(status + 1 + b, 1u);
                if (prev == (unsigned)(S * Hkv) - 1u) {
                    if (fits) seq_len[b] = L0 + n_new;
                    atomicExch(status + 1 + b, 0u);
                }
            }
        }
    };
    const int S_pages = S - ((n_sink + n_recent > 0) ? 2 : 0);   // the last two splits take the tier
    uint8_t *slots = unit_slots(const_cast<uint8_t *>(pages), gridDim.z, Hkv, NB, 2, unit, n_sink + n_recent, NG);
    if (s >= S_pages) {
        after_prep();
        if (BK) {
            __syncthreads();
            tier_cta_q(sh, slots, len, n_sink, n_recent, s - S_pages, k,
                       TierQBuckets{qsel, idx + unit * nbk * k, k, nbk, w_pages * kT, qrow0}, part_o, part_ml,
                       qrow0, S, s, out, counters + unit, rot);
        } else {
            load_sel(0);
            tier_cta(sh, slots, len, n_sink, n_recent, s - S_pages, k, part_o, part_ml, qrow0, S, s, out,
                     counters + unit, rot);
        }
        return;
    }
    const Tier tr = tier_of(len, n_sink, n_recent);
    const uint8_t *unit_pages = pages + unit * NB * (size_t)page_bytes(2, NG);
    if constexpr (BK) {
        after_prep();
        if constexpr (STEP)
            run_pages<NG, false>(sh, unit_pages, tr.sink_end, tr.recent_start,
                                 split_of(tr.recent_start, S_pages, s), Pool{}, S, s, qrow0, part_o, part_ml, out,
                                 counters + unit, status, polls, rot, w_pages, load_plan);
        else
            run_pages<NG, false>(sh, unit_pages, tr.sink_end, tr.recent_start,
                                 split_of(tr.recent_start, S_pages, s), Pool{}, S, s, qrow0, part_o, part_ml, out,
                                 counters + unit, status, polls, rot, w_pages, load_sel);
    } else {
        // the tails of the pair's first two pages (while they hold no new
        // token) are copied, and their key rows brought into L2, before the
        // channel choice is in place
        Pool pool = unit_pool(tr.sink_end, tr.recent_start, s, warp >> 1, S_pages);
        for (int j = 0; j < 2; j++) {
            const int qj = pool.index(j);
            if (qj < 0 || (STEP && pool.page(qj) >= L0 / kT)) break;
            pool.pre = j + 1;
        }
        if ((tid & 63) == 0) {
            for (int j = 0; j < pool.pre; j++) {
                const uint8_t *pg = unit_pages + (size_t)pool.page(pool.index(j)) * page_bytes(2, NG);
                issue_tail<NG>(sh, warp >> 1, j, pg);
                prefetch_l2(pg, kKeyBytes);
            }
        }
        after_prep();
        if constexpr (STEP)
            load_plan(0);
        else
            load_sel(0);
        run_pages<NG, true>(sh, unit_pages, tr.sink_end, tr.recent_start, Split{0, 0}, pool, S, s, qrow0, part_o,
                            part_ml, out, counters + unit, status, polls, rot, 0, [](int) {});
    }
}

// ---------------------------------------------------------------- fused step
__device__ __forceinline__ void cluster_arrive() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
    asm volatile("barrier.cluster.wait.acquire.aligned;\n" ::: "memory");
}

static_assert(4 * kD == 2 * kThreads, "two query elements per thread");
template <typename Tin, int NG>
__global__ void __cluster_dims__(kCluster, 1, 1) __launch_bounds__(kThreads, 2)
step_mma_kernel(uint8_t *__restrict__ pages, int32_t *__restrict__ seq_len, uint32_t *__restrict__ status,
                int Hkv, int NB, int Hq, const Tin *__restrict__ q, const Tin *__restrict__ k_new,
                const Tin *__restrict__ v_new, int n_new, const double *__restrict__ A,
                const double *__restrict__ Ainvt, const double *__restrict__ delta,
                const double *__restrict__ v_rot, double vclip, int k, int32_t *__restrict__ idx, float *__restrict__ qsel,
                float *__restrict__ qgsum, float *__restrict__ part_o, float2 *__restrict__ part_ml, int S,
                float *__restrict__ out, int n_sink, int n_recent) {
    namespace cg = cooperative_groups;
    extern __shared__ __align__(16) uint8_t smem_raw[];
    MmaShared &sh = *reinterpret_cast<MmaShared *>(smem_raw);
    uint8_t *P = &sh.stage[0][0][0];
    double (*a_hi)[kCols] = reinterpret_cast<double (*)[kCols]>(P + kOffAHi);   // A[64 + ., 64r + .]
    double (*a_lo)[kCols] = reinterpret_cast<double (*)[kCols]>(P + kOffALo);   // A[., 64r + .]
    double *e2 = reinterpret_cast<double *>(P + kOffE2);
    int (*rank_part)[kD] = reinterpret_cast<int (*)[kD]>(P + kOffRank);
    double (*qp)[kD] = reinterpret_cast<double (*)[kD]>(P + kOffQp);
    PexScratch &px = *reinterpret_cast<PexScratch *>(&sh.pex[0][0][0]);
    float *ks_f = &sh.q[0][0];                                                   // [nw][128]
    double (*ks)[kD] = reinterpret_cast<double (*)[kD]>(P + kOffKs);             // [nw][128], later
    double (*vsd)[kD] = reinterpret_cast<double (*)[kD]>(P + kOffVs);            // [nw][128], later

    cg::cluster_group cluster = cg::this_cluster();
    const int r = (int)cluster.block_rank();        // channels 64r..64r+63
    const int s = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int B = gridDim.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const size_t unit = (size_t)b * Hkv + h;
    const size_t qrow0 = (size_t)b * Hq + (size_t)h * 4;
    uint8_t *unit_pages = pages + unit * NB * (size_t)page_bytes(2, NG);
    const int capacity = NB * kT;
    const int NPt = n_sink + n_recent;
    const int S_pages = S - (NPt > 0 ? kCluster : 0);
    const bool is_tier = s >= S_pages;
    // the first cluster holds the new tokens' pages and the tier cluster
    // writes what no split reads: only these may append
    const bool may_append = is_tier || s < kCluster;
    // 64-column block of a 128 x 128 float64 matrix: 128 rows of 512 bytes
    auto stage_block = [&](double (*dst)[kCols], const double *src, int row0, int rows) {
        for (int e = tid; e < rows * (kBlkRowBytes / 16); e += kThreads) {
            const int c = e >> 5, part = e & 31;
            cp_async16(&dst[c][2 * part], src + (size_t)(row0 + c) * kD + 2 * part);
        }
    };
    // rows 32p..32p+7 and 32p+8..32p+31 of the staged A^{-T} block
    auto ai_base = [&](int p, int upper) -> uint8_t * {
        if (may_append) return P + (32 * p + 8 * upper) * kBlkRowBytes;
        return upper ? sh.stage[p][1] : sh.stage[p][0];
    };

    // every global read that does not depend on the length is issued first,
    // so that the prologue waits for one round trip: the A^{-T} block, the
    // query, and in the CTAs that may append, A's low rows and the new rows
    if (tid < kD) sh.chan_pos[tid] = -1;
    if (tid < 2 * kPairs) mbar_init(smem_u32(&sh.mbar[tid >> 1][tid & 1]), 1);
    // the length and the query first: small, and what the first barrier waits for
    if (tid == 0) sh.s_len = seq_len[b];
    double qv[2];
#pragma unroll
    for (int i = 0; i < 2; i++) qv[i] = in_to_double(q[qrow0 * kD + tid + i * kThreads]);
    const double *Ai_blk = Ainvt + (size_t)h * kD * kD + r * kCols;
    const double *A_blk = A + (size_t)h * kD * kD + r * kCols;
    // one commit group per 32 rows, so the chains start on the first rows
#pragma unroll 1
    for (int p = 0; p < 4; p++) {
        for (int e = tid; e < 32 * (kBlkRowBytes / 16); e += kThreads) {
            const int rr = e >> 5, part = e & 31, c = 32 * p + rr;
            double *row = reinterpret_cast<double *>(ai_base(p, rr >= 8) + (rr < 8 ? rr : rr - 8) * kBlkRowBytes);
            cp_async16(row + 2 * part, Ai_blk + (size_t)c * kD + 2 * part);
        }
        cp_async_commit();
    }
    const int nload = may_append ? min(n_new, kStepMaxNew) : 0;   // new rows this CTA may need
    float vpre[kVPre];
    if (nload > 0) {
        stage_block(a_lo, A_blk, 0, 64);            // a fifth commit group
        const size_t in0 = unit * (size_t)n_new;
        for (int e = tid; e < nload * kD; e += kThreads) ks_f[e] = in_to_float(k_new[in0 * kD + e]);
#pragma unroll
        for (int i = 0; i < kVPre; i++) {
            const int e = tid + i * kThreads;
            vpre[i] = e < nload * kD ? in_to_float(v_new[in0 * kD + e]) : 0.f;
        }
    }
    cp_async_commit();
#pragma unroll
    for (int i = 0; i < 2; i++) {
        const int e = tid + i * kThreads;
        px.qin[e % kD][e / kD] = qv[i];
    }
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    __syncthreads();

    // new length (a step that would overflow the capacity appends nothing and
    // raises KVQ_DEV_CAPACITY, like kvq_append) and this pair's page pool;
    // with a protected tier the last cluster reads the BF16 slots instead of
    // pages, and the pages cover the coded tokens [sink_end, recent_start)
    const int L0 = sh.s_len;
    const bool ok = L0 >= 0 && L0 + n_new <= capacity;
    const int len = min(max(ok ? L0 + n_new : L0, 0), capacity);
    const Tier tr = tier_of(len, n_sink, n_recent);
    Pool pool = unit_pool(tr.sink_end, tr.recent_start, s, warp >> 1, S_pages);
    pool.appenders = min(kPairs * kCluster, pool.NP);
    pool.skip = pool.appenders < pool.NP ? kAppendRounds : 0;
    pool.pre = may_append ? 0 : 1;
    // the first page's tail (no new token in it) is copied while the channels
    // are chosen
    if (!is_tier && !may_append && (tid & 63) == 0 && pool.index(0) >= 0) {
        const uint8_t *first = unit_pages + (size_t)pool.page(pool.index(0)) * page_bytes(2, NG);
        issue_tail<NG>(sh, warp >> 1, 0, first);
        prefetch_l2(first, kKeyBytes);          // the key rows: in L2 once the choice is made
    }
    // New tokens w in [w0, w1) are transformed here: in the first cluster,
    // those whose pages are in the pool (its pairs read them first, after the
    // append), or -- all of them -- in the tier cluster, which writes their
    // BF16 slots and the codes of pages no split reads in this step.
    int w0 = 0, w1 = 0;
    if (ok && n_new > 0) {
        if (is_tier) {
            w1 = n_new;
        } else if (s < kCluster) {
            for (int w = 0; w < n_new; w++)
                if ((L0 + w) / kT < pool.P1) w1 = w + 1;
        }
    }
    const int nw = w1 - w0;           // w0 = 0: the rows loaded above are tokens 0..nw-1
    // every CTA of sequence b has read its length once the counter reaches
    // S * Hkv; the last one stores the new length
    if (tid == 0) {
        if (!ok && s == 0 && h == 0) atomicOr(status, (uint32_t)KVQ_DEV_CAPACITY);
        const unsigned prev = atomicAdd(status + 1 + b, 1u);
        if (prev == (unsigned)(S * Hkv) - 1u) {
            if (ok) seq_len[b] = L0 + n_new;
            atomicExch(status + 1 + b, 0u);
        }
    }
    // q'[hl][64r + jj] = sum_c q[hl][c] Ainvt[c][64r + jj], fma chain c =
    // 0..127 from 0.0, the four heads' chains side by side in thread jj (each
    // A^{-T} element loaded once), each 32-row group as soon as it has landed,
    // the operands loaded four steps ahead; then the pooled energy of channel
    // 64r + jj, with a diagonal refinement of the base queries q'_{h,j} /
    // delta_j (the arithmetic of kvq_select_channels)
    double acc[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll 1
    for (int p = 0; p < 4; p++) {
        cp_async_wait_upto(3 - p + (nload > 0 ? 1 : 0));
        __syncthreads();
        if (tid < kCols) {
            const double *lo8 = reinterpret_cast<const double *>(ai_base(p, 0));
            const double *hi24 = reinterpret_cast<const double *>(ai_base(p, 1));
            auto arow = [&](int rr) { return rr < 8 ? lo8[rr * kCols + tid] : hi24[(rr - 8) * kCols + tid]; };
            double a[4];
            double2 qa[4], qb[4];
#pragma unroll
            for (int u = 0; u < 4; u++) {
                a[u] = arow(u);
                qa[u] = *reinterpret_cast<const double2 *>(&px.qin[32 * p + u][0]);
                qb[u] = *reinterpret_cast<const double2 *>(&px.qin[32 * p + u][2]);
            }
#pragma unroll
            for (int rr = 0; rr < 32; rr++) {
                const int u = rr & 3;
                acc[0] = fma(qa[u].x, a[u], acc[0]);
                acc[1] = fma(qa[u].y, a[u], acc[1]);
                acc[2] = fma(qb[u].x, a[u], acc[2]);
                acc[3] = fma(qb[u].y, a[u], acc[3]);
                if (rr + 4 < 32) {
                    a[u] = arow(rr + 4);
                    qa[u] = *reinterpret_cast<const double2 *>(&px.qin[32 * p + rr + 4][0]);
                    qb[u] = *reinterpret_cast<const double2 *>(&px.qin[32 * p + rr + 4][2]);
                }
            }
        }
    }
    if (nload > 0) cp_async_wait<0>();              // A's low rows (read after the barrier below)
    if (tid < kCols) {
        const double dj = delta ? delta[(size_t)h * kD + r * kCols + tid] : 1.0;
        double e = 0.0;
#pragma unroll
        for (int hl = 0; hl < 4; hl++) {
            sh.qp_own[hl][tid] = acc[hl];
            const double u = delta ? acc[hl] / dj : acc[hl];
            e = fma(u, u, e);
        }
        sh.e2_own[tid] = e;
    }
    __syncthreads();                                // A^{-T} block no longer needed
    if (nw > 0) {
        // K'[t][j] = sum_c K[t][c] A[c][j], fma chain c = 0..127 from 0.0, for
        // token w0 + warp / 2 and channel j = 64r + jj: rows 0..63 of A while
        // rows 64..127 are staged
        stage_block(a_hi, A_blk, 64, 64);
        cp_async_commit();
        for (int e = tid; e < nw * kD; e += kThreads) ks[e / kD][e % kD] = (double)ks_f[e];
#pragma unroll
        for (int i = 0; i < kVPre; i++) {
            const int e = tid + i * kThreads;
            if (e < nw * kD) vsd[e / kD][e % kD] = (double)vpre[i];
        }
        __syncthreads();
        const int w = warp >> 1, jj = (warp & 1) * 32 + lane, j = r * kCols + jj;
        const double *R_blk = v_rot ? v_rot + (size_t)h * kD * kD + r * kCols : nullptr;
        double x = 0.0;
        if (w < nw) {
#pragma unroll 16
            for (int c = 0; c < 64; c++) x = fma(ks[w][c], a_lo[c][jj], x);
        }
        cp_async_wait<0>();
        __syncthreads();
        if (R_blk) {                                // rows 0..63 of the rotation over A's
            stage_block(a_lo, R_blk, 0, 64);
            cp_async_commit();
        }
        if (w < nw) {                               // uniform over the warp
#pragma unroll 16
            for (int c = 64; c < kD; c++) x = fma(ks[w][c], a_hi[c - 64][jj], x);
        }
        // value of channel j: (V Rv)[j] by the same chain with the rotation in
        // place of A, or V[j]
        double v = w < nw ? vsd[w][j] : 0.0;
        if (R_blk) {
            __syncthreads();                        // every read of A's high rows is done
            stage_block(a_hi, R_blk, 64, 64);
            cp_async_commit();
            cp_async_wait<1>();
            __syncthreads();
            double y = 0.0;
            if (w < nw) {
#pragma unroll 16
                for (int c = 0; c < 64; c++) y = fma(vsd[w][c], a_lo[c][jj], y);
            }
            cp_async_wait<0>();
            __syncthreads();
            if (w < nw) {
#pragma unroll 16
                for (int c = 64; c < kD; c++) y = fma(vsd[w][c], a_hi[c - 64][jj], y);
            }
            v = y;
        }
        if (w < nw) {                               // uniform over the warp
            const int pos = L0 + w0 + w;
            if (is_tier && stores_slot(pos, L0 + n_new, n_sink, n_recent)) {
                uint16_t *dst = reinterpret_cast<uint16_t *>(unit_slots(pages, B, Hkv, NB, 2, unit, NPt, NG) +
                                                             (size_t)slot_of(pos, n_sink, n_recent) * kSlotBytes);
                dst[j] = __bfloat16_as_ushort(__double2bfloat16(x));
                dst[kD + j] = __bfloat16_as_ushort(__double2bfloat16(v));
            }
        }
        // codes: by the cluster of the page, or by the tier cluster when no
        // split reads the page in this step (uniform over the warp).  Groups
        // of 32: warp = group; one grid per token: the range of token w is
        // met over warps 2w, 2w+1 of both CTAs (distributed shared memory).
        double klo = 0.0, khi = 0.0, vlo = 0.0, vhi = 0.0;
        if constexpr (NG == 1) {
            if (w < nw) {
                const double a = warp_min(j != 0 ? x : pos_inf()), bk = warp_max(j != 0 ? x : neg_inf());
                const double c = warp_min(v), d = warp_max(v);
                if (lane == 0) {
                    sh.trange[warp][0] = a;
                    sh.trange[warp][1] = bk;
                    sh.trange[warp][2] = c;
                    sh.trange[warp][3] = d;
                }
            }
            cluster.sync();
            if (w < nw) {
                const MmaShared *peer = cluster.map_shared_rank(&sh, r ^ 1);
                const int w2 = warp & ~1;
                klo = fmin(fmin(sh.trange[w2][0], sh.trange[w2 + 1][0]), fmin(peer->trange[w2][0], peer->trange[w2 + 1][0]));
                khi = fmax(fmax(sh.trange[w2][1], sh.trange[w2 + 1][1]), fmax(peer->trange[w2][1], peer->trange[w2 + 1][1]));
                vlo = fmin(fmin(sh.trange[w2][2], sh.trange[w2 + 1][2]), fmin(peer->trange[w2][2], peer->trange[w2 + 1][2]));
                vhi = fmax(fmax(sh.trange[w2][3], sh.trange[w2 + 1][3]), fmax(peer->trange[w2][3], peer->trange[w2 + 1][3]));
            }
        }
        if (w < nw && (!is_tier || (L0 + w0 + w) / kT >= pool.P1)) {
            const int g = NG == 1 ? 0 : 2 * r + (warp & 1);                  // metadata group
            const bool meta_writer = NG == 1 ? (r == 0 && (warp & 1) == 0 && lane == 0) : lane == 0;
            const int pos = L0 + w0 + w, tt = pos % kT;
            uint8_t *page = unit_pages + (size_t)(pos / kT) * page_bytes(2, NG);
            uint16_t sb, zb;
            const uint32_t kc = NG == 1 ? code_in_range<2>(x, klo, khi, sb, zb) : quantize_lane<2>(x, j != 0, sb, zb);
            if (meta_writer)
                reinterpret_cast<uint32_t *>(page + off_kmeta(2))[meta_word(g, tt)] = (uint32_t)sb | ((uint32_t)zb << 16);
            if (j == 0) reinterpret_cast<uint16_t *>(page + off_ch0(2))[tt] = __bfloat16_as_ushort(__double2bfloat16(x));
            const uint32_t vc = NG == 1 ? code_in_range<2>(v, __dmul_rn(vclip, vlo), __dmul_rn(vclip, vhi), sb, zb)
                                        : quantize_lane<2>(v, true, sb, zb, vclip);
            if (meta_writer)
                reinterpret_cast<uint32_t *>(page + off_vmeta(2, NG))[meta_word(g, tt)] = (uint32_t)sb | ((uint32_t)zb << 16);
            // positions at or beyond the stored length hold zero bits, so the
            // codes are OR-ed in (the other new tokens share the words)
            const int word = tt / 16, shf = 2 * (tt % 16);
            if (j != 0) atomicOr(reinterpret_cast<uint32_t *>(page + (size_t)j * row_bytes(2)) + word, kc << shf);
            atomicOr(reinterpret_cast<uint32_t *>(page + off_vcodes(2) + (size_t)j * row_bytes(2)) + word, vc << shf);
            // the page is read next through the async proxy (bulk copies)
            asm volatile("fence.proxy.async.global;\n" ::: "memory");
        }
    }
    __syncthreads();
    cluster.sync();            // the cluster's q', energies and new tokens are in place
    // the 128 energies and all of q', this CTA's half and the peer's (each
    // thread's five values loaded before it stores any)
    double my_q[4] = {0.0, 0.0, 0.0, 0.0};
    if (tid < kD) {
        const MmaShared *peer = cluster.map_shared_rank(&sh, tid / kCols);
        const int l = tid % kCols;
        const double my_e = peer->e2_own[l];
#pragma unroll
        for (int hl = 0; hl < 4; hl++) my_q[hl] = peer->qp_own[hl][l];
        e2[tid] = my_e;
#pragma unroll
        for (int hl = 0; hl < 4; hl++) qp[hl][tid] = my_q[hl];
    }
    __syncthreads();
    cluster_arrive();          // done reading the other CTA's shared memory (waited for at exit)

    // ---- channel choice (the arithmetic of kvq_select_channels)
    {
        // rank of channel j among 1..127 by (energy descending, index
        // ascending), in two halves
        const int j = tid & (kD - 1), part = tid >> 7;
        rank_part[part][j] = rank_half(reinterpret_cast<const unsigned long long *>(e2), j, part);
    }
    __syncthreads();
    if (tid < kD) {
        const bool sel = (tid == 0) || (rank_part[0][tid] + rank_part[1][tid] < k - 1);
        const unsigned m = __ballot_sync(0xffffffffu, sel);
        if (lane == 0) sh.selmask[warp] = m;
    }
    __syncthreads();
    // Everything else follows from the 128-bit choice mask, in parallel:
    // warps 0..3 the list positions, fp32 q' and the outputs; warp 4 the
    // zero-point sums; warp 5 the copy list; every warp one k-step's B
    // fragments.
    uint32_t msk[4];
#pragma unroll
    for (int w = 0; w < 4; w++) msk[w] = sh.selmask[w];
    auto selected = [&](int c) {
        const uint32_t m = c < 64 ? (c < 32 ? msk[0] : msk[1]) : (c < 96 ? msk[2] : msk[3]);
        return (m >> (c & 31)) & 1u;
    };
    if (tid < kD) {
        const uint32_t mw = warp < 2 ? (warp == 0 ? msk[0] : msk[1]) : (warp == 2 ? msk[2] : msk[3]);
        if ((mw >> lane) & 1u) {
            int pos = __popc(mw & ((1u << lane) - 1u));
#pragma unroll
            for (int w = 0; w < 3; w++) pos += w < warp ? __popc(msk[w]) : 0;
            sh.chan_pos[tid] = pos;
#pragma unroll
            for (int hl = 0; hl < 4; hl++) {
                const float qf = (float)my_q[hl];
                sh.q[hl][pos] = qf;
                if (tid == 0) sh.plan.q0[hl] = qf;      // channel 0 is position 0
                if (s == 0) qsel[(qrow0 + hl) * k + pos] = qf;
            }
            if (s == 0) idx[unit * k + pos] = tid;
        }
    } else if (warp == 4 && lane < 4 * kNG) {
        // zero-point sum of key group gr (channel 0 is bf16, not in group 0),
        // kept channels ascending from 0.0 (a kept channel adds fma(1, q', s)
        // = s + q' exactly, a dropped one fma(0, q', s) = s); one grid per
        // token: entry 0 sums every channel, the others are 0
        const int hl = lane / kNG, gr = lane % kNG;
        constexpr int GS = kD / NG;                 // channels per key group
        double sm = 0.0;
        if (gr < NG)
            for (int c = (gr == 0 ? 1 : gr * GS); c < (gr + 1) * GS; c++)
                sm = fma(selected(c) ? 1.0 : 0.0, qp[hl][c], sm);
        const float gf = (float)sm;
        sh.plan.qg[hl][gr] = gf;
        if (s == 0) qgsum[(qrow0 + hl) * kNG + gr] = gf;
    } else if (warp == 5) {
        // the copy list of a page
        plan_copies_warp(sh.plan, plan_chunks(msk), NG, lane);
    }
    {
        // score-MMA B fragments of k-step `warp`: channel 0 and unselected
        // channels get q' = 0
        auto qf = [&](int hh, int c) -> float { return (c >= 1 && selected(c)) ? (float)qp[hh][c] : 0.f; };
        sh.plan.bq[warp][lane] = make_uint2(plan_bq_word(warp, lane, 0, qf), plan_bq_word(warp, lane, 1, qf));
    }
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    __syncthreads();

    const double *rot = v_rot ? v_rot + (size_t)h * kD * kD : nullptr;
    if (is_tier)
        tier_cta(sh, unit_slots(pages, B, Hkv, NB, 2, unit, NPt, NG), len, n_sink, n_recent, s - S_pages, k, part_o,
                 part_ml, qrow0, S, s, out, status + 1 + B + unit, rot);
    else
        run_pages<NG, true>(sh, unit_pages, tr.sink_end, tr.recent_start, Split{0, 0}, pool, S, s, qrow0, part_o,
                            part_ml, out, status + 1 + B + unit, status, kWaitPolls, rot, 0, [](int) {});
    cluster_wait();            // the other CTA no longer reads this CTA's shared memory
}

}  // namespace

// Splits per (sequence, KV head): about two CTAs per SM in all (counting the
// `tier` CTAs that handle the protected tier), at most one page split per
// kPairs pages, at least one.  Returns page splits + tier.
int decode_mma_splits(int units, int nblk, int num_sms, int tier) {
    int S = (2 * num_sms) / units - tier;
    const int max_s = nblk / kPairs;
    if (S > max_s) S = max_s;
    return (S < 1 ? 1 : S) + tier;
}

uint32_t default_wait_polls() { return kWaitPolls; }

template <int NG, bool BK, bool STEP>
cudaError_t launch_decode_mma_t(const kvq_cache &c, int Hq, const int32_t *idx, const float *qsel,
                                const float *qgsum, int k, float *part_o, float2 *part_ml, int S,
                                float *out, uint32_t polls, int n_new, const PagePlan *plans, cudaStream_t st) {
    const size_t smem = sizeof(MmaShared);
    static std::atomic<uint64_t> done{0};
    cudaError_t e = set_smem_once(decode_mma_kernel<NG, BK, STEP>, (int)smem, done);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)S, (unsigned)c.n_kv_heads, (unsigned)c.batch);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    // a step's decode may start while the preparation kernel still runs
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = STEP ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, decode_mma_kernel<NG, BK, STEP>, static_cast<const uint8_t *>(c.pages),
                              c.seq_len, (int)c.n_kv_heads, c.capacity / kT, Hq, idx, qsel, qgsum, k, part_o,
                              part_ml, S, out, unit_counter(c, 0, 0), c.status, (int)c.n_sink, (int)c.n_recent,
                              c.v_rot, buckets_of(c), c.bucket / kT, polls, n_new, plans);
}

template <bool STEP>
cudaError_t launch_decode_mma_any(const kvq_cache &c, int Hq, const int32_t *idx, const float *qsel,
                                  const float *qgsum, int k, float *part_o, float2 *part_ml, int S, float *out,
                                  uint32_t polls, int n_new, const PagePlan *plans, cudaStream_t st) {
    const bool one = groups_of(c) == 1, bk = c.bucket > 0;
    if (bk)
        return one ? launch_decode_mma_t<1, true, STEP>(c, Hq, idx, qsel, qgsum, k, part_o, part_ml, S, out, polls,
                                                        n_new, plans, st)
                   : launch_decode_mma_t<kNG, true, STEP>(c, Hq, idx, qsel, qgsum, k, part_o, part_ml, S, out,
                                                          polls, n_new, plans, st);
    return one ? launch_decode_mma_t<1, false, STEP>(c, Hq, idx, qsel, qgsum, k, part_o, part_ml, S, out, polls,
                                                     n_new, plans, st)
               : launch_decode_mma_t<kNG, false, STEP>(c, Hq, idx, qsel, qgsum, k, part_o, part_ml, S, out, polls,
                                                       n_new, plans, st);
}

cudaError_t launch_decode_mma(const kvq_cache &c, int Hq, const int32_t *idx, const float *qsel,
                              const float *qgsum, int k, float *part_o, float2 *part_ml, int S,
                              float *out, uint32_t polls, cudaStream_t st) {
    return launch_decode_mma_any<false>(c, Hq, idx, qsel, qgsum, k, part_o, part_ml, S, out, polls, 0, nullptr, st);
}

// The decode of a step whose preparation kernel (the channel choices, the
// page plans `plans` and the append of n_new tokens) was launched just before
// it on `st`.
cudaError_t launch_decode_mma_step(const kvq_cache &c, int Hq, const int32_t *idx, const float *qsel,
                                   const float *qgsum, int k, float *part_o, float2 *part_ml, int S,
                                   float *out, int n_new, const PagePlan *plans, cudaStream_t st) {
    return launch_decode_mma_any<true>(c, Hq, idx, qsel, qgsum, k, part_o, part_ml, S, out, kWaitPolls, n_new,
                                       plans, st);
}

template <typename Tin, int NG>
cudaError_t launch_step_mma_t(const kvq_cache &c, int Hq, const void *q, const void *k_new, const void *v_new,
                              int n_new, const double *A, const double *Ainvt, const double *delta, int k,
                              int32_t *idx, float *qsel, float *qgsum, float *part_o, float2 *part_ml, int S,
                              float *out, cudaStream_t st) {
    const size_t smem = sizeof(MmaShared);
    static std::atomic<uint64_t> done{0};
    cudaError_t e = set_smem_once(step_mma_kernel<Tin, NG>, (int)smem, done);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)S, (unsigned)c.n_kv_heads, (unsigned)c.batch);
    step_mma_kernel<Tin, NG><<<grid, kThreads, smem, st>>>(
        static_cast<uint8_t *>(c.pages), c.seq_len, c.status, c.n_kv_heads, c.capacity / kT, Hq,
        static_cast<const Tin *>(q), static_cast<const Tin *>(k_new), static_cast<const Tin *>(v_new), n_new, A,
        Ainvt, delta, c.v_rot, value_clip(c), k, idx, qsel, qgsum, part_o, part_ml, S, out, c.n_sink, c.n_recent);
    return cudaGetLastError();
}

// The whole decode step in one launch (no RoPE buckets).
cudaError_t launch_step_mma(const kvq_cache &c, int Hq, const void *q, const void *k_new, const void *v_new,
                            int dtype, int n_new, const double *A, const double *Ainvt, const double *delta,
                            int k, int32_t *idx, float *qsel, float *qgsum, float *part_o, float2 *part_ml,
                            int S, float *out, cudaStream_t st) {
    const bool one = groups_of(c) == 1;
    if (dtype == KVQ_DTYPE_F32)
        return one ? launch_step_mma_t<float, 1>(c, Hq, q, k_new, v_new, n_new, A, Ainvt, delta, k, idx, qsel,
                                                 qgsum, part_o, part_ml, S, out, st)
                   : launch_step_mma_t<float, kNG>(c, Hq, q, k_new, v_new, n_new, A, Ainvt, delta, k, idx, qsel,
                                                   qgsum, part_o, part_ml, S, out, st);
    return one ? launch_step_mma_t<uint16_t, 1>(c, Hq, q, k_new, v_new, n_new, A, Ainvt, delta, k, idx, qsel,
                                                qgsum, part_o, part_ml, S, out, st)
               : launch_step_mma_t<uint16_t, kNG>(c, Hq, q, k_new, v_new, n_new, A, Ainvt, delta, k, idx, qsel,
                                                  qgsum, part_o, part_ml, S, out, st);
}

int step_mma_max_new() { return kStepMaxNew; }
int step_mma_cluster() { return kCluster; }

size_t decode_mma_smem_bytes() { return sizeof(MmaShared); }

}  // namespace kvq
