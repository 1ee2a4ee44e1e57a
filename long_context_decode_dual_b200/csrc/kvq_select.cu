// kvq_select_channels: query transform and top-k channel choice.
//
// "Dual-QK: Sharp Queries and Flat Keys for Prunable 2-bit KV Caches":
//   §3.1 the query is multiplied by the inverse transpose of the key
//        transform, so transformed scores equal the original ones;
//   §3.2 Eq. 4: channel energy pooled over the query heads sharing a KV head,
//        e_j^2 = sum_h q'_{h,j}^2, one mask per KV head, chosen per query;
//   §3.3, App. C.2: with a diagonal refinement D folded into the transforms
//        the energies are those of the base queries, q'_{h,j} / delta_j;
//   §3.4: with bucket-relative RoPE each bucket that holds a token gets its
//        own choice, made on the query moved into the bucket's frame (its
//        anchor's rotary rotation removed).
// Channel 0 is always kept; ties go to the lower channel index.
//
// One thread-block cluster of four CTAs = one (sequence, KV head) and a run
// of up to nbb consecutive RoPE buckets (one bucket without RoPE); CTA r owns
// channels 32r..32r+31 (key group r).  The kernel is built for latency: every
// read that does not depend on the length goes out at once (its 32 columns of
// A^{-T}, 32 KB, as four groups of 32 rows; the query), the query is moved
// into each bucket's frame, and the fixed-order fp64 fma chains q'_b[h][j] of
// its channels start on the first 32 rows while the rest arrive, the chains
// of four query rows side by side in one thread (one A^{-T} load for the
// four), then their pooled energies.  After a cluster barrier every CTA reads
// the four energy blocks of every bucket through distributed shared memory
// and ranks its own 32 channels by energy among all 128 (eight threads per
// channel, exact integer compares); after a second barrier each CTA reads
// the others' 32-bit keep masks, so all four hold the same 128-bit choice.
// Each writes the outputs of its own channels: their list positions (prefix
// counts of the per-bucket masks), q' in fp32 and its group's zero-point sum.  Buckets past
// the sequence's length (other than bucket 0) are skipped.  Before a
// tensor-core decode the kernel also writes each bucket's page plan (the
// decode's score-MMA operands and copy list).
//
// Decode-step preparation (APPEND): the same kernel also appends the step's
// new tokens -- the arithmetic of kvq_append, in the first cluster of each
// (sequence, KV head), where CTA r owns key and value channels 32r..32r+31
// just as for the query.  A's columns (and the value rotation's) are staged
// with A^{-T}'s; warp 4 + w runs token w's key chain (and value chain), lane
// = channel, beside the query chains, then quantizes and writes the codes,
// metadata, channel 0 and protected slots.  The sequence length is not
// advanced here: the decode kernel that follows (launched as a programmatic
// dependent, so that it starts streaming its first pages while this kernel
// runs) advances it once it has waited for this grid.  A decode step with RoPE
// buckets runs the append in the small-append kernel before this one instead
// (StepAppend::here = 0): this kernel then makes the choice for the length
// with the new tokens, starts as that kernel's programmatic dependent, and
// waits for it before exiting, so its own completion implies the append's.
#include "kvq_internal.cuh"

#include <cooperative_groups.h>

namespace kvq {
namespace {

namespace cg = cooperative_groups;

constexpr int kThreads = 256;
constexpr int kCtas = kNG;                 // CTAs per cluster, one per key group
constexpr int kMaxGNbb = 32;               // heads x buckets of one cluster

__device__ __forceinline__ void cluster_arrive_release() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void cluster_wait_acquire() {
    asm volatile("barrier.cluster.wait.acquire.aligned;\n" ::: "memory");
}

// Dynamic shared memory of one CTA (doubles, then ints): the 32-column
// blocks of A^{-T} (As) and, when appending, of A (Ab) and the value
// rotation (Rb), each [128][32]; the query rows in each bucket's frame,
// transposed, qT[128][Rp] (row = bucket * g + head, Rp = R rounded up to 4);
// the query as loaded, qin[g][128] (with RoPE only); q' of this CTA's
// channels qp[R][32]; energies e2own[nbb][32] and e2s[nbb][128]; the new
// rows ks[4][128], vs[4][128] and the ranges trange[4][4][4] (CTA, token,
// {key lo, hi, value lo, hi}); words mask[nbb][4]; bytes sel[nbb][128],
// rank[nbb][32][8] (this CTA's channels' partial ranks) and the new tokens'
// codes codes[4][64] (key, value).
constexpr int kPrepMaxNew = 4;
struct SelLayout {
    int g, nbb;
    bool app, rot, rope;
    __host__ __device__ int R() const { return g * nbb; }
    __host__ __device__ int Rp() const { return (R() + 3) & ~3; }
    __host__ __device__ int off_Ab() const { return kD * kGroup; }
    __host__ __device__ int off_Rb() const { return off_Ab() + (app ? kD * kGroup : 0); }
    __host__ __device__ int off_qT() const { return off_Rb() + (rot ? kD * kGroup : 0); }
    __host__ __device__ int off_qin() const { return off_qT() + kD * Rp(); }
    __host__ __device__ int off_qp() const { return off_qin() + (rope ? g * kD : 0); }
    __host__ __device__ int off_e2own() const { return off_qp() + Rp() * kGroup; }
    __host__ __device__ int off_e2s() const { return off_e2own() + nbb * kGroup; }
    __host__ __device__ int off_ks() const { return off_e2s() + nbb * kD; }
    __host__ __device__ int off_vs() const { return off_ks() + (app ? kPrepMaxNew * kD : 0); }
    __host__ __device__ int off_tr() const { return off_vs() + (app ? kPrepMaxNew * kD : 0); }
    __host__ __device__ int end_doubles() const { return off_tr() + (app ? kCtas * kPrepMaxNew * 4 : 0); }
    __host__ __device__ size_t bytes() const {
        return (size_t)end_doubles() * sizeof(double) + (size_t)nbb * (4 * sizeof(uint32_t) + 3 * kD) +
               (app ? kPrepMaxNew * 2 * kGroup : 0);
    }
};

// The step's new tokens for the preparation kernel (APPEND).
struct StepAppend {
    uint8_t *pages;
    uint32_t *status;             // the cache's status word (also without an append)
    const void *K, *V;            // [B][Hkv][n_new][128] of the input dtype
    const double *A, *Rv;         // [Hkv][128][128]; Rv may be null
    double vclip;
    int n_new, NB, capacity, n_sink, n_recent;
    int here;                     // 1: this kernel appends; 0: the kernel before it does (this one is
                                  // its programmatic dependent and waits for it before exiting)
};

constexpr uint32_t kPrepPolls = 1u << 20;         // bound on the polls of one wait for a row group

// wait (bounded) until a row group's copies have landed (phase 0)
__device__ __forceinline__ void drain_bar(uint32_t bar) {
    for (uint32_t i = 0; i < kPrepPolls; i++)
        if (mbar_try_wait(bar, 0u)) return;
}

template <typename Tin, bool APPEND, int NG>
__global__ void __cluster_dims__(kCtas, 1, 1) __launch_bounds__(kThreads)
select_kernel(const Tin *__restrict__ q, const double *__restrict__ Ainvt, const double *__restrict__ delta,
              int Hq, int Hkv, int g, int k, int32_t *__restrict__ idx, float *__restrict__ qsel,
              float *__restrict__ qgsum, int ng, const int32_t *__restrict__ seq_len,
              const double *__restrict__ rope, int nbk, int w, int nbb, StepAppend ap,
              PagePlan *__restrict__ plans) {
    extern __shared__ __align__(16) double sm[];
    const bool app_here = APPEND && ap.here;        // this kernel writes the new tokens
    const SelLayout L{g, nbb, app_here, app_here && ap.Rv != nullptr, rope != nullptr};
    const int Rp = L.Rp();
    double *As = sm;
    double *Ab = sm + L.off_Ab();
    double *Rb = sm + L.off_Rb();
    double *qT = sm + L.off_qT();
    double *qin = sm + L.off_qin();
    double *qp = sm + L.off_qp();
    double *e2own = sm + L.off_e2own();
    double *e2s = sm + L.off_e2s();
    double *ks = sm + L.off_ks();
    double *vs = sm + L.off_vs();
    double *trange = sm + L.off_tr();
    uint32_t *mask = reinterpret_cast<uint32_t *>(sm + L.end_doubles());   // [nbb][4]
    uint8_t *sel = reinterpret_cast<uint8_t *>(mask + nbb * 4);           // [nbb][128]
    uint8_t *rank = sel + nbb * kD;                                       // [nbb][32][8], each <= 16
    uint8_t *codes = rank + 2 * nbb * kD;                                 // [token][key 32, value 32]

    if constexpr (APPEND) asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
    cg::cluster_group cluster = cg::this_cluster();
    const int r = (int)cluster.block_rank();        // = blockIdx.x % 4
    const int b0 = (blockIdx.x / kCtas) * nbb;       // first bucket of the cluster
    const int h = blockIdx.y, b = blockIdx.z, t = threadIdx.x;
    const int lane = t & 31, warp = t >> 5;
    const size_t qrow0 = (size_t)b * Hq + (size_t)h * g;
    const size_t unit = (size_t)b * Hkv + h;
    const int j = r * kGroup + lane;                 // this lane's key / value channel
    const bool first = b0 == 0;                      // the cluster that appends

    // Every read that does not depend on the length goes out first: the
    // column blocks (A^{-T}; A and the value rotation in the first cluster),
    // one bulk copy per 256-byte row, completing on the mbarrier of its group
    // of 32 rows; the query and the new rows; then the length.
    __shared__ uint64_t grp_bar[4];
    const double *Ai = Ainvt + (size_t)h * kD * kD;
    const double *Ah = app_here ? ap.A + (size_t)h * kD * kD : nullptr;
    const bool stage_a = app_here && first;
    const double *Rh = (stage_a && ap.Rv) ? ap.Rv + (size_t)h * kD * kD : nullptr;
    constexpr uint32_t kRowBytes = kGroup * sizeof(double);
    if (t < 4) {
        mbar_init(smem_u32(&grp_bar[t]), 1);
        mbar_arrive_expect_tx(smem_u32(&grp_bar[t]), 32u * kRowBytes * (1u + (stage_a ? 1u : 0u) + (Rh ? 1u : 0u)));
    }
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    __syncthreads();
    if (t < kD) {
        const uint32_t bar = smem_u32(&grp_bar[t / 32]);
        bulk_g2s(smem_u32(As + t * kGroup), Ai + (size_t)t * kD + r * kGroup, kRowBytes, bar);
        if (Rh) bulk_g2s(smem_u32(Rb + t * kGroup), Rh + (size_t)t * kD + r * kGroup, kRowBytes, bar);
    } else if (stage_a) {
        const int c = t - kD;
        bulk_g2s(smem_u32(Ab + c * kGroup), Ah + (size_t)c * kD + r * kGroup, kRowBytes, smem_u32(&grp_bar[c / 32]));
    }
    bool gave_up = false;                            // a wait for a row group gave up (KVQ_DEV_TIMEOUT)
    const int aw = warp - kThreads / 64;             // new token of this warp (warps 4..7 append)
    double vnew = 0.0;                               // the value of (token aw, channel j)
    if constexpr (APPEND) {
        if (stage_a && ap.n_new > 0) {
            const Tin *Kn = static_cast<const Tin *>(ap.K), *Vn = static_cast<const Tin *>(ap.V);
            const size_t in_base = unit * (size_t)ap.n_new;
            for (int e = t; e < ap.n_new * kD; e += kThreads) {
                ks[e] = in_to_double(Kn[in_base * kD + e]);
                if (Rh) vs[e] = in_to_double(Vn[in_base * kD + e]);
            }
            if (aw >= 0 && aw < ap.n_new) vnew = in_to_double(Vn[(in_base + aw) * kD + j]);
        }
    }
    double *q_dst = rope ? qin : qT;                 // without RoPE the one "bucket" is the query itself
    for (int e = t; e < g * kD; e += kThreads) {
        const int hl = e / kD, c = e % kD;
        const double v = in_to_double(q[qrow0 * kD + e]);
        if (rope) q_dst[e] = v;                      // [hl][c]
        else q_dst[c * Rp + hl] = v;                 // [c][row]
    }
    // the step's new tokens: appended by the first cluster of the unit; the
    // choice is made for the length once they are in (a step that would
    // overflow the capacity appends nothing)
    const int L0 = seq_len[b];
    const bool ok = !APPEND || (L0 >= 0 && L0 + ap.n_new <= ap.capacity);
    const bool appends = stage_a && ok;
    // buckets that hold a token (bucket 0 always): a prefix of the buckets
    const int len = max(APPEND && ok ? L0 + ap.n_new : L0, 0);
    const int used = rope ? max(1, (int)(((long long)len + w - 1) / w)) : 1;
    const int nb = min(min(nbb, nbk - b0), used - b0);   // buckets of this cluster to do
    if (nb <= 0) {                                      // the whole cluster
        if (t < 4) drain_bar(smem_u32(&grp_bar[t]));     // no copy may land after the exit
        return;
    }
    if (APPEND && first && !ok && t == 0) atomicOr(ap.status, (uint32_t)KVQ_DEV_CAPACITY);
    // The new tokens' code bits are merged into their rows by one thread per
    // row (threads 128..159 key rows, 160..191 value rows of channels
    // 32r..32r+31), which loads the row's words that the new positions fall
    // in now (at most two: the tokens are consecutive) and stores them after
    // the codes are known; only this kernel writes them in this step.
    const int mrow = t - kThreads / 2;               // 0..63 on the merge threads
    const bool merger = APPEND && appends && ap.n_new > 0 && mrow >= 0 && mrow < 2 * kGroup &&
                        (mrow >= kGroup || r * kGroup + mrow != 0);     // channel 0's key row is unused
    uint32_t *mw0 = nullptr, *mw1 = nullptr;         // the words of the first and the last new token
    uint32_t mv0 = 0u, mv1 = 0u;
    if (merger) {
        uint8_t *unit_pg = ap.pages + unit * ap.NB * (size_t)page_bytes(2, NG);
        const size_t roff = (mrow >= kGroup ? (size_t)off_vcodes(2) : 0) +
                            (size_t)(r * kGroup + mrow % kGroup) * row_bytes(2);
        const int p0 = L0, p1 = L0 + ap.n_new - 1;
        mw0 = reinterpret_cast<uint32_t *>(unit_pg + (size_t)(p0 / kT) * page_bytes(2, NG) + roff) + (p0 % kT) / 16;
        mw1 = reinterpret_cast<uint32_t *>(unit_pg + (size_t)(p1 / kT) * page_bytes(2, NG) + roff) + (p1 % kT) / 16;
        mv0 = *mw0;
        if (mw1 != mw0) mv1 = *mw1;
    }
    __syncthreads();                                 // query and new rows in place
    if (rope) {
        // q T_b for each bucket: channel pairs (i, i + 64) rotated back by the anchor's angle
        const double2 *cs = reinterpret_cast<const double2 *>(rope);
        for (int e = t; e < nb * g * (kD / 2); e += kThreads) {
            const int bi = e / (g * (kD / 2)), rem = e % (g * (kD / 2));
            const int hl = rem / (kD / 2), i = rem % (kD / 2);
            double x0 = qin[hl * kD + i], x1 = qin[hl * kD + i + kD / 2];
            rope_unanchor_pair(x0, x1, __ldg(cs + (size_t)(b0 + bi) * (kD / 2) + i));
            qT[i * Rp + bi * g + hl] = x0;
            qT[(i + kD / 2) * Rp + bi * g + hl] = x1;
        }
        if (appends) {
            // k T_b for the bucket of each new position
            for (int e = t; e < ap.n_new * (kD / 2); e += kThreads) {
                const int i = e / (kD / 2), c = e % (kD / 2);
                rope_unanchor_pair(ks[i * kD + c], ks[i * kD + c + kD / 2],
                                   __ldg(cs + (size_t)((L0 + i) / w) * (kD / 2) + c));
            }
        }
        __syncthreads();                             // the rows in the buckets' frames in place
    }

    // Chains, fma over c = 0..127 from 0.0, row block p as soon as it has
    // landed: q'_b[hl][j] = sum_c qT_b[c][hl] Ainvt[c][j], rows 4w..4w+3 of
    // the query rows in warp w (one A^{-T} load for the four); K'[aw][j] =
    // sum_c K[aw][c] A[c][j] and, with a value rotation, (V Rv)[aw][j] in
    // warp 4 + aw.
    const int row0 = 4 * warp;
    const bool has_q = row0 < nb * g;
    const bool has_k = appends && aw >= 0 && aw < ap.n_new;
    const bool has_v = has_k && Rh != nullptr;
    double acc[4] = {0.0, 0.0, 0.0, 0.0};
    double xk = 0.0, xv = 0.0;
    const int rq = min(row0, Rp - 4);                // rows read (clamped into the buffer)
    // each step's operands are loaded four steps ahead (the fma chains run
    // at their own latency, not the shared-memory loads')
#pragma unroll 1
    for (int p = 0; p < 4; p++) {
        if (has_q || has_k) {
            if (!mbar_wait_bounded(smem_u32(&grp_bar[p]), 0u, ap.status, kPrepPolls)) gave_up = true;
        }
        if (has_q) {
            double a[4];
            double2 qa[4], qb[4];
#pragma unroll
            for (int u = 0; u < 4; u++) {
                const int c = 32 * p + u;
                a[u] = As[c * kGroup + lane];
                qa[u] = *reinterpret_cast<const double2 *>(qT + c * Rp + rq);
                qb[u] = *reinterpret_cast<const double2 *>(qT + c * Rp + rq + 2);
            }
#pragma unroll
            for (int cc = 0; cc < 32; cc++) {
                const int u = cc & 3;
                acc[0] = fma(qa[u].x, a[u], acc[0]);
                acc[1] = fma(qa[u].y, a[u], acc[1]);
                acc[2] = fma(qb[u].x, a[u], acc[2]);
                acc[3] = fma(qb[u].y, a[u], acc[3]);
                if (cc + 4 < 32) {
                    const int c = 32 * p + cc + 4;
                    a[u] = As[c * kGroup + lane];
                    qa[u] = *reinterpret_cast<const double2 *>(qT + c * Rp + rq);
                    qb[u] = *reinterpret_cast<const double2 *>(qT + c * Rp + rq + 2);
                }
            }
        }
        if (has_k) {
            double kx[4], ka[4], vx[4], va[4];
#pragma unroll
            for (int u = 0; u < 4; u++) {
                const int c = 32 * p + u;
                kx[u] = ks[aw * kD + c];
                ka[u] = Ab[c * kGroup + lane];
                vx[u] = has_v ? vs[aw * kD + c] : 0.0;
                va[u] = has_v ? Rb[c * kGroup + lane] : 0.0;
            }
#pragma unroll
            for (int cc = 0; cc < 32; cc++) {
                const int u = cc & 3;
                xk = fma(kx[u], ka[u], xk);
                xv = fma(vx[u], va[u], xv);
                if (cc + 4 < 32) {
                    const int c = 32 * p + cc + 4;
                    kx[u] = ks[aw * kD + c];
                    ka[u] = Ab[c * kGroup + lane];
                    vx[u] = has_v ? vs[aw * kD + c] : 0.0;
                    va[u] = has_v ? Rb[c * kGroup + lane] : 0.0;
                }
            }
        }
    }
    if (has_v) vnew = xv;
    if (has_q) {
#pragma unroll
        for (int u = 0; u < 4; u++) {
            const int row = rq + u;
            if (row >= row0 && row < nb * g) qp[row * kGroup + lane] = acc[u];   // [bi * g + hl][lane]
        }
    }
    // one grid per token: this CTA's share of each new token's key and value
    // ranges, met over the cluster after the barrier below
    if (NG == 1 && has_k) {
        const double a = warp_min(j != 0 ? xk : pos_inf()), bk = warp_max(j != 0 ? xk : neg_inf());
        const double c = warp_min(vnew), d = warp_max(vnew);
        if (lane == 0) {
            double *tr = trange + (r * kPrepMaxNew + aw) * 4;
            tr[0] = a;
            tr[1] = bk;
            tr[2] = c;
            tr[3] = d;
        }
    }
    __syncthreads();
    // e_j^2 per bucket, fma chain over heads ascending from 0.0; with a
    // diagonal refinement D, of the base queries q'_{h,j} / delta_j
    for (int e = t; e < nb * kGroup; e += kThreads) {
        const int bi = e / kGroup, l = e % kGroup;
        const double dj = delta ? delta[(size_t)h * kD + r * kGroup + l] : 1.0;
        double en = 0.0;
        for (int hl = 0; hl < g; hl++) {
            const double v = qp[(bi * g + hl) * kGroup + l];
            const double u = delta ? v / dj : v;
            en = fma(u, u, en);
        }
        e2own[e] = en;
    }
    cluster.sync();                                // every CTA's energies (and ranges) are ready
    // everything read from the other CTAs, in one pass: the energies; with
    // one grid per token, the new tokens' ranges, and in CTA 0 all of q' (for
    // the zero-point sums) into the query buffer, no longer needed
    for (int e = t; e < nb * kD; e += kThreads) {
        const int bi = e / kD, jj = e % kD;
        const double *src = cluster.map_shared_rank(e2own, jj / kGroup);
        e2s[e] = src[bi * kGroup + jj % kGroup];
    }
    double *qall = qT;                                 // [R][128]
    if (NG == 1 && appends && t < kCtas * kPrepMaxNew * 4) {
        // CTA rr's ranges sit in its own slot rr, the only slot the others
        // read; this CTA fills its other slots from them
        const int rr = t / (kPrepMaxNew * 4);
        if (rr != r) trange[t] = cluster.map_shared_rank(trange, rr)[t];
    }
    if (ng != kNG && r == 0) {
        for (int e = t; e < nb * g * kD; e += kThreads) {
            const int row = e / kD, c = e % kD;
            qall[e] = cluster.map_shared_rank(qp, c / kGroup)[row * kGroup + c % kGroup];
        }
    }
    __syncthreads();
    // Per bucket, the rank of each of this CTA's 32 channels among 1..127 by
    // (energy descending, index ascending), counted in eight parts of 16
    // channels by eight threads; channel 0 and the k - 1 channels of rank
    // below k - 1 are kept.  The CTA's 32 keep bits go to its slot of the
    // buckets' 128-bit masks, which the CTAs then read from one another.
    for (int e = t; e < nb * kGroup * 8; e += kThreads) {
        const int bi = e / (kGroup * 8), l = (e / 8) % kGroup, part = e % 8;
        rank[e] = (uint8_t)rank_count<16>(reinterpret_cast<const unsigned long long *>(e2s + bi * kD),
                                          r * kGroup + l, 16 * part);
    }
    __syncthreads();
    for (int e = t; e < nb * kGroup; e += kThreads) {  // whole warps: one warp per bucket
        const int bi = e / kGroup, l = e % kGroup, c = r * kGroup + l;
        int rk = 0;
#pragma unroll
        for (int part = 0; part < 8; part++) rk += rank[e * 8 + part];
        const unsigned m = __ballot_sync(0xffffffffu, c == 0 || rk < k - 1);
        if (l == 0) mask[bi * 4 + r] = m;
    }
    cluster.sync();                                // every CTA's keep bits are in place
    for (int e = t; e < nb * 4; e += kThreads) {
        // CTA rr's bits sit in its own slot rr, the only slot the others read
        const int rr = e % 4;
        if (rr != r) mask[e] = cluster.map_shared_rank(mask, rr)[e];
    }
    __syncthreads();
    cluster_arrive_release();                        // done reading the other CTAs (waited for at exit)
    for (int e = t; e < nb * kD; e += kThreads) {
        const int bi = e / kD, jj = e % kD;
        sel[e] = (uint8_t)((mask[bi * 4 + jj / 32] >> (jj % 32)) & 1u);
    }
    __syncthreads();
    // Outputs, by warp role (a role's loop wraps onto the next threads when it
    // has more tasks): warps 0-1 this CTA's channels' list positions, channel
    // numbers and fp32 q'; warp 2 the zero-point sums; warp 3 the plans' copy
    // lists and channel 0; warps 4-7 the new tokens' codes and the plans' B
    // fragments.
    for (int e = t; e < nb * kGroup; e += kThreads) {
        const int bi = e / kGroup, l = e % kGroup, c = r * kGroup + l;
        if (!sel[bi * kD + c]) continue;
        int pos = __popc(mask[bi * 4 + r] & ((1u << l) - 1u));
        for (int m = 0; m < r; m++) pos += __popc(mask[bi * 4 + m]);
        const int bk = b0 + bi;
        idx[(unit * nbk + bk) * k + pos] = c;
        for (int hl = 0; hl < g; hl++)
            qsel[((qrow0 + hl) * nbk + bk) * k + pos] = (float)qp[(bi * g + hl) * kGroup + l];
    }
    // zero-point sum of each key group (channel 0 is bf16, not in group 0),
    // kept channels ascending from 0.0: groups of 32 -- CTA r sums group r;
    // one grid per token -- CTA 0 sums all channels into entry 0, the rest
    // are 0
    for (int e = (t + kThreads - 64) % kThreads; e < nb * g; e += kThreads) {
        const int bi = e / g, hl = e % g;
        double s = 0.0;
        if (ng == kNG) {
            for (int l = (r == 0 ? 1 : 0); l < kGroup; l++)
                if (sel[bi * kD + r * kGroup + l]) s += qp[(bi * g + hl) * kGroup + l];
        } else if (r == 0) {
            const double *qrow = qall + (bi * g + hl) * kD;
            for (int c = 1; c < kD; c++)
                if (sel[bi * kD + c]) s += qrow[c];
        } else {
            continue;
        }
        float *o = qgsum + ((qrow0 + hl) * nbk + b0 + bi) * kNG;
        float *pg = plans ? plans[unit * nbk + b0 + bi].qg[hl] : nullptr;
        if (ng == kNG) {
            o[r] = (float)s;
            if (pg) pg[r] = (float)s;
        } else {
#pragma unroll
            for (int gr = 0; gr < kNG; gr++) {
                o[gr] = gr == 0 ? (float)s : 0.f;
                if (pg) pg[gr] = gr == 0 ? (float)s : 0.f;
            }
        }
    }
    // the page plans of the tensor-core decode that follows (four heads):
    // CTA r writes the score-MMA B fragments of its channels (k-steps 2r and
    // 2r + 1) and its group's zero-point sums (above); CTA 0 channel 0's q'
    // and the copy lists
    if (plans) {
        if (r == 0 && warp == 3) {
            for (int bi = 0; bi < nb; bi++) {
                const uint32_t msk[4] = {mask[bi * 4], mask[bi * 4 + 1], mask[bi * 4 + 2], mask[bi * 4 + 3]};
                PagePlan &pl = plans[unit * nbk + b0 + bi];
                plan_copies_warp(pl, plan_chunks(msk), NG, lane);
                if (lane < 4) pl.q0[lane] = (float)qp[(bi * 4 + lane) * kGroup];
            }
        }
        for (int e = (t + kThreads - 128) % kThreads; e < nb * 64; e += kThreads) {
            const int bi = e / 64, ks2 = 2 * r + (e / 32) % 2, ln = e % 32;
            auto qf = [&](int hh, int c) -> float {
                return (c >= 1 && sel[bi * kD + c]) ? (float)qp[(bi * 4 + hh) * kGroup + (c - r * kGroup)] : 0.f;
            };
            plans[unit * nbk + b0 + bi].bq[ks2][ln] = make_uint2(plan_bq_word(ks2, ln, 0, qf),
                                                                 plan_bq_word(ks2, ln, 1, qf));
        }
    }
    if constexpr (APPEND) {
        // the new tokens' codes, metadata, channel 0 and protected slots (the
        // arithmetic of kvq_append)
        if (has_k) {                                 // uniform over the warp
            uint8_t *unit_pg = ap.pages + unit * ap.NB * (size_t)page_bytes(2, NG);
            double klo = 0.0, khi = 0.0, vlo = 0.0, vhi = 0.0;
            if constexpr (NG == 1) {
                klo = pos_inf(), khi = neg_inf(), vlo = pos_inf(), vhi = neg_inf();
#pragma unroll
                for (int rr = 0; rr < kCtas; rr++) {
                    const double *pr = trange + (rr * kPrepMaxNew + aw) * 4;
                    klo = fmin(klo, pr[0]);
                    khi = fmax(khi, pr[1]);
                    vlo = fmin(vlo, pr[2]);
                    vhi = fmax(vhi, pr[3]);
                }
            }
            const int pos = L0 + aw, tt = pos % kT;
            uint8_t *page = unit_pg + (size_t)(pos / kT) * page_bytes(2, NG);
            const int mg = NG == 1 ? 0 : r;                  // metadata group
            const bool meta_writer = lane == 0 && (NG != 1 || r == 0);
            uint16_t sb, zb;
            const uint32_t kc = NG == 1 ? code_in_range<2>(xk, klo, khi, sb, zb) : quantize_lane<2>(xk, j != 0, sb, zb);
            if (meta_writer)
                reinterpret_cast<uint32_t *>(page + off_kmeta(2))[meta_word(mg, tt)] = (uint32_t)sb | ((uint32_t)zb << 16);
            if (j == 0) reinterpret_cast<uint16_t *>(page + off_ch0(2))[tt] = __bfloat16_as_ushort(__double2bfloat16(xk));
            const uint32_t vc =
                NG == 1 ? code_in_range<2>(vnew, __dmul_rn(ap.vclip, vlo), __dmul_rn(ap.vclip, vhi), sb, zb)
                        : quantize_lane<2>(vnew, true, sb, zb, ap.vclip);
            if (meta_writer)
                reinterpret_cast<uint32_t *>(page + off_vmeta(2, NG))[meta_word(mg, tt)] = (uint32_t)sb | ((uint32_t)zb << 16);
            codes[aw * 2 * kGroup + lane] = (uint8_t)kc;
            codes[aw * 2 * kGroup + kGroup + lane] = (uint8_t)vc;
            if (ap.n_sink + ap.n_recent > 0 && stores_slot(pos, L0 + ap.n_new, ap.n_sink, ap.n_recent)) {
                uint16_t *dst = reinterpret_cast<uint16_t *>(
                    unit_slots(ap.pages, gridDim.z, Hkv, ap.NB, 2, unit, ap.n_sink + ap.n_recent, NG) +
                    (size_t)slot_of(pos, ap.n_sink, ap.n_recent) * kSlotBytes);
                dst[j] = __bfloat16_as_ushort(__double2bfloat16(xk));
                dst[kD + j] = __bfloat16_as_ushort(__double2bfloat16(vnew));
            }
        }
        __syncthreads();
        if (merger) {
            // clear each new token's 2-bit field and set its code, in order
            for (int i = 0; i < ap.n_new; i++) {
                const int pos = L0 + i, shf = 2 * (pos % 16);
                const uint32_t c = (uint32_t)codes[i * 2 * kGroup + mrow] << shf;
                if (pos / 16 == L0 / 16)
                    mv0 = (mv0 & ~(3u << shf)) | c;
                else
                    mv1 = (mv1 & ~(3u << shf)) | c;
            }
            *mw0 = mv0;
            if (mw1 != mw0) *mw1 = mv1;
        }
    }
    // after a give-up, no copy may land once the CTA has exited
    if (__syncthreads_or(gave_up) && t < 4) drain_bar(smem_u32(&grp_bar[t]));
    // the step's append ran in the kernel before this one: this grid
    // completes only after it, so the decode that waits for this grid sees
    // the new tokens
    if (APPEND && !ap.here) asm volatile("griddepcontrol.wait;\n" ::: "memory");
    cluster_wait_acquire();                          // no other CTA still reads this one's shared memory
}

template <typename Tin, bool APPEND, int NG>
cudaError_t launch_select_t(const kvq_cache &c, const void *q, int Hq, const double *Ainvt, const double *delta,
                            int k, int32_t *idx, float *qsel, float *qgsum, const StepAppend &ap, PagePlan *plans,
                            cudaStream_t st) {
    const int g = Hq / c.n_kv_heads;
    const int nbk = buckets_of(c);
    const double *rope = c.bucket > 0 ? c.rope : nullptr;
    const int nbb = rope ? std::min(nbk, std::max(1, kMaxGNbb / g)) : 1;     // buckets per cluster
    const bool here = APPEND && ap.here;
    const SelLayout L{g, nbb, here, here && ap.Rv != nullptr, rope != nullptr};
    // the largest layout any call can ask for (g <= 32, g * nbb <= 32 or nbb =
    // 1; the step's preparation only for four query heads per KV head)
    size_t max_smem = 0;
    for (int gg = APPEND ? 4 : 1; gg <= (APPEND ? 4 : 32); gg++)
        for (int rp = 0; rp < 2; rp++) {
            const SelLayout Lg{gg, rp ? std::max(1, kMaxGNbb / gg) : 1, APPEND, APPEND, rp != 0};
            max_smem = std::max(max_smem, Lg.bytes());
        }
    static std::atomic<uint64_t> done{0};
    cudaError_t e = set_smem_once(select_kernel<Tin, APPEND, NG>, (int)max_smem, done);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(kCtas * ((nbk + nbb - 1) / nbb)), (unsigned)c.n_kv_heads, (unsigned)c.batch);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = L.bytes();
    cfg.stream = st;
    // after the step's append kernel: start while it runs (programmatic
    // dependent launch); the kernel waits for it before it exits
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = (APPEND && !ap.here) ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, select_kernel<Tin, APPEND, NG>, static_cast<const Tin *>(q), Ainvt, delta, Hq,
                              (int)c.n_kv_heads, g, k, idx, qsel, qgsum, groups_of(c),
                              static_cast<const int32_t *>(c.seq_len), rope, nbk, (int)c.bucket, nbb, ap, plans);
}

}  // namespace

cudaError_t launch_select(const kvq_cache &c, const void *q, int dtype, int Hq, const double *Ainvt,
                          const double *delta, int k, int32_t *idx, float *qsel, float *qgsum, cudaStream_t st) {
    StepAppend none{};
    none.status = c.status;                          // for the bounded waits' KVQ_DEV_TIMEOUT
    none.here = 1;
    return dtype == KVQ_DTYPE_F32
               ? launch_select_t<float, false, kNG>(c, q, Hq, Ainvt, delta, k, idx, qsel, qgsum, none, nullptr, st)
               : launch_select_t<uint16_t, false, kNG>(c, q, Hq, Ainvt, delta, k, idx, qsel, qgsum, none, nullptr,
                                                       st);
}

// The first launch of a decode step (INT2, four query heads per KV head, at
// most 4 new tokens): the channel choice of kvq_select_channels, the page
// plans of the decode, and the append of kvq_append without the length
// advance; it lets the next launch on the stream start early (programmatic
// dependent launch).
cudaError_t launch_step_prep(const kvq_cache &c, const void *q, int dtype, int Hq, const void *k_new,
                             const void *v_new, int n_new, const double *A, const double *Ainvt,
                             const double *delta, int k, int32_t *idx, float *qsel, float *qgsum, PagePlan *plans,
                             bool append_here, cudaStream_t st) {
    const StepAppend ap{static_cast<uint8_t *>(c.pages), c.status, k_new, v_new, A, c.v_rot, value_clip(c), n_new,
                        c.capacity / kT, c.capacity, c.n_sink, c.n_recent, append_here ? 1 : 0};
    const bool one = groups_of(c) == 1;
    if (dtype == KVQ_DTYPE_F32)
        return one ? launch_select_t<float, true, 1>(c, q, Hq, Ainvt, delta, k, idx, qsel, qgsum, ap, plans, st)
                   : launch_select_t<float, true, kNG>(c, q, Hq, Ainvt, delta, k, idx, qsel, qgsum, ap, plans, st);
    return one ? launch_select_t<uint16_t, true, 1>(c, q, Hq, Ainvt, delta, k, idx, qsel, qgsum, ap, plans, st)
               : launch_select_t<uint16_t, true, kNG>(c, q, Hq, Ainvt, delta, k, idx, qsel, qgsum, ap, plans, st);
}
int step_prep_max_new() { return kPrepMaxNew; }

}  // namespace kvq
