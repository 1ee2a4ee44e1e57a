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
// channels 32r..32r+31 (key group r).  It stages its 32 columns of A^{-T}
// (32 KB) once with one cp.async burst, moves the query into each bucket's
// frame, and runs the fixed-order fp64 fma chains q'_b[h][j] of its channels
// for every bucket (four independent chains per thread at a time), then their
// pooled energies.  After a cluster barrier every CTA reads the four energy
// blocks of every bucket through distributed shared memory and makes the same
// exact choice (a bitonic sort per bucket, one warp each, in registers), so
// no CTA waits for another's decision; each writes the outputs of its own
// channels: their list positions (prefix counts of per-bucket 128-bit
// masks), q' in fp32 and its group's zero-point sum.  Buckets past the
// sequence's length (other than bucket 0) are skipped.
//
// Decode-step preparation (APPEND): the same kernel also appends the step's
// new tokens -- the arithmetic of kvq_append, in the first cluster of each
// (sequence, KV head), where CTA r owns key and value channels 32r..32r+31
// just as for the query.  Warps 4..7, idle in the query chains of four heads,
// run the new tokens' key chains (warp 4 + w = token w, lane = channel) while
// warps 0..3 run the query's, then quantize and write the codes, metadata,
// channel 0 and protected slots.  The sequence length is not advanced here:
// the decode kernel that follows (launched as a programmatic dependent, so
// that it starts streaming its first pages while this kernel runs) advances
// it once it has waited for this grid.
#include "kvq_internal.cuh"

#include <cooperative_groups.h>

namespace kvq {
namespace {

namespace cg = cooperative_groups;

constexpr int kThreads = 256;
constexpr int kCtas = kNG;                 // CTAs per cluster, one per key group
constexpr int kMaxGNbb = 32;               // heads x buckets of one cluster

// Dynamic shared memory of one CTA: doubles As[128][32], qin[g][128],
// qr[nbb][g][128] (the query in each bucket's frame), qp[nbb][g][32],
// e2own[nbb][32], e2s[nbb][128]; then ints sel[nbb][128] and words
// mask[nbb][4].
struct SelLayout {
    int g, nbb;
    __host__ __device__ int off_qin() const { return kD * kGroup; }
    __host__ __device__ int off_qr() const { return off_qin() + g * kD; }
    __host__ __device__ int off_qp() const { return off_qr() + nbb * g * kD; }
    __host__ __device__ int off_e2own() const { return off_qp() + nbb * g * kGroup; }
    __host__ __device__ int off_e2s() const { return off_e2own() + nbb * kGroup; }
    __host__ __device__ int end_doubles() const { return off_e2s() + nbb * kD; }
    __host__ __device__ size_t bytes() const {
        return (size_t)end_doubles() * sizeof(double) + (size_t)nbb * (kD + 4) * sizeof(int);
    }
};
// Append scratch of the preparation kernel, after SelLayout (16-byte aligned):
// the CTA's 32 columns of A (then of the value rotation), the new key and
// value rows in float64, the ranges of one grid per token, and the codes.
constexpr int kPrepMaxNew = 4;
struct PrepScratch {
    double Ab[kD][kGroup];
    double ks[kPrepMaxNew][kD];
    double vsd[kPrepMaxNew][kD];
    double trange[kPrepMaxNew][4];
    uint8_t kcode[kPrepMaxNew][kGroup];
    uint8_t vcode[kPrepMaxNew][kGroup];
    int s_len;
};
__host__ __device__ inline size_t prep_offset(const SelLayout &L) { return (L.bytes() + 15) & ~(size_t)15; }

// The step's new tokens for the preparation kernel (APPEND).
struct StepAppend {
    uint8_t *pages;
    uint32_t *status;
    const void *K, *V;            // [B][Hkv][n_new][128] of the input dtype
    const double *A, *Rv;         // [Hkv][128][128]; Rv may be null
    double vclip;
    int n_new, NB, capacity, n_sink, n_recent;
};

template <typename Tin, bool APPEND, int NG>
__global__ void __cluster_dims__(kCtas, 1, 1) __launch_bounds__(kThreads)
select_kernel(const Tin *__restrict__ q, const double *__restrict__ Ainvt, const double *__restrict__ delta,
              int Hq, int Hkv, int g, int k, int32_t *__restrict__ idx, float *__restrict__ qsel,
              float *__restrict__ qgsum, int ng, const int32_t *__restrict__ seq_len,
              const double *__restrict__ rope, int nbk, int w, int nbb, StepAppend ap) {
    extern __shared__ __align__(16) double sm[];
    const SelLayout L{g, nbb};
    double *As = sm;
    double *qin = sm + L.off_qin();
    double *qr = rope ? sm + L.off_qr() : qin;       // without RoPE the one "bucket" is the query itself
    double *qp = sm + L.off_qp();
    double *e2own = sm + L.off_e2own();
    double *e2s = sm + L.off_e2s();
    int *sel = reinterpret_cast<int *>(sm + L.end_doubles());
    uint32_t *mask = reinterpret_cast<uint32_t *>(sel + nbb * kD);

    if constexpr (APPEND) asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
    cg::cluster_group cluster = cg::this_cluster();
    const int r = (int)cluster.block_rank();        // = blockIdx.x % 4
    const int b0 = (blockIdx.x / kCtas) * nbb;       // first bucket of the cluster
    const int h = blockIdx.y, b = blockIdx.z, t = threadIdx.x;
    const int lane = t & 31, warp = t >> 5;
    const size_t qrow0 = (size_t)b * Hq + (size_t)h * g;
    // the step's new tokens: appended by the first cluster of the unit; the
    // choice is made for the length once they are in (a step that would
    // overflow the capacity appends nothing)
    const int L0 = seq_len[b];
    const bool ok = !APPEND || (L0 >= 0 && L0 + ap.n_new <= ap.capacity);
    const bool appends = APPEND && b0 == 0 && ok;
    // buckets that hold a token (bucket 0 always): a prefix of the buckets
    const int len = max(APPEND && ok ? L0 + ap.n_new : L0, 0);
    const int used = rope ? max(1, (int)(((long long)len + w - 1) / w)) : 1;
    const int nb = min(min(nbb, nbk - b0), used - b0);   // buckets of this cluster to do
    if (nb <= 0) return;                                // the whole cluster
    if (APPEND && b0 == 0 && !ok && t == 0) atomicOr(ap.status, (uint32_t)KVQ_DEV_CAPACITY);

    // columns 32r..32r+31 of A^{-T} for this KV head: 128 rows of 256 bytes
    const double *Ai = Ainvt + (size_t)h * kD * kD + r * kGroup;
    for (int e = t; e < kD * kGroup / 2; e += kThreads) {
        const int c = e >> 4, part = e & 15;
        cp_async16(As + c * kGroup + 2 * part, Ai + (size_t)c * kD + 2 * part);
    }
    PrepScratch *px = nullptr;
    const int aw = warp - kThreads / 64;             // new token of this warp (warps 4..7 append)
    const int j = r * kGroup + lane;                 // this lane's key / value channel
    double vnew = 0.0;                               // the value of (token aw, channel j)
    if constexpr (APPEND) {
        px = reinterpret_cast<PrepScratch *>(reinterpret_cast<uint8_t *>(sm) + prep_offset(L));
        if (appends) {
            // the same 32 columns of A, and the new rows
            const double *Ah = ap.A + (size_t)h * kD * kD + r * kGroup;
            for (int e = t; e < kD * kGroup / 2; e += kThreads) {
                const int c = e >> 4, part = e & 15;
                cp_async16(&px->Ab[c][2 * part], Ah + (size_t)c * kD + 2 * part);
            }
            const Tin *Kn = static_cast<const Tin *>(ap.K), *Vn = static_cast<const Tin *>(ap.V);
            const size_t in_base = ((size_t)b * Hkv + h) * (size_t)ap.n_new;
            for (int e = t; e < ap.n_new * kD; e += kThreads) {
                px->ks[e / kD][e % kD] = in_to_double(Kn[in_base * kD + e]);
                if (ap.Rv) px->vsd[e / kD][e % kD] = in_to_double(Vn[in_base * kD + e]);
            }
            if (aw >= 0 && aw < ap.n_new) vnew = in_to_double(Vn[(in_base + aw) * kD + j]);
        }
    }
    cp_async_commit();
    for (int e = t; e < g * kD; e += kThreads) qin[e] = in_to_double(q[qrow0 * kD + e]);
    __syncthreads();
    if (APPEND && appends && rope) {
        // k T_b for the bucket of each new position
        const double2 *cs = reinterpret_cast<const double2 *>(rope);
        for (int e = t; e < ap.n_new * (kD / 2); e += kThreads) {
            const int i = e / (kD / 2), c = e % (kD / 2);
            rope_unanchor_pair(px->ks[i][c], px->ks[i][c + kD / 2], __ldg(cs + (size_t)((L0 + i) / w) * (kD / 2) + c));
        }
    }
    if (rope) {
        // q T_b for each bucket: channel pairs (i, i + 64) rotated back by the anchor's angle
        const double2 *cs = reinterpret_cast<const double2 *>(rope);
        for (int e = t; e < nb * g * (kD / 2); e += kThreads) {
            const int bi = e / (g * (kD / 2)), rem = e % (g * (kD / 2));
            const int hl = rem / (kD / 2), i = rem % (kD / 2);
            double x0 = qin[hl * kD + i], x1 = qin[hl * kD + i + kD / 2];
            rope_unanchor_pair(x0, x1, __ldg(cs + (size_t)(b0 + bi) * (kD / 2) + i));
            qr[(bi * g + hl) * kD + i] = x0;
            qr[(bi * g + hl) * kD + i + kD / 2] = x1;
        }
    }
    cp_async_wait<0>();
    __syncthreads();

    // q'_b[hl][j] = sum_c qr_b[hl][c] Ainvt[c][j], fma chain c = 0..127 from
    // 0.0; task (bi, hl, lane), four independent chains per thread at a time
    const int ntask = nb * g * kGroup;
    for (int t0 = t; t0 < ntask; t0 += 4 * kThreads) {
        double acc[4] = {0.0, 0.0, 0.0, 0.0};
        const double *qrow[4];
#pragma unroll
        for (int u = 0; u < 4; u++) {
            const int task = min(t0 + u * kThreads, ntask - 1);
            qrow[u] = qr + (task / kGroup) * kD;          // row (bi * g + hl)
        }
#pragma unroll 8
        for (int c = 0; c < kD; c++) {
            const double a = As[c * kGroup + lane];
#pragma unroll
            for (int u = 0; u < 4; u++) acc[u] = fma(qrow[u][c], a, acc[u]);
        }
#pragma unroll
        for (int u = 0; u < 4; u++) {
            const int task = t0 + u * kThreads;
            if (task < ntask) qp[task] = acc[u];          // [bi][hl][lane]
        }
    }
    // the new tokens' keys, K'[aw][j] = sum_c K[aw][c] A[c][j] (fma chain c =
    // 0..127 from 0.0), then with a value rotation (V Rv)[aw][j] by the same
    // chain with Rv's columns staged over A's
    double xnew = 0.0;
    if constexpr (APPEND) {
        const bool mine = appends && aw >= 0 && aw < ap.n_new;
        if (mine) {
#pragma unroll 16
            for (int c = 0; c < kD; c++) xnew = fma(px->ks[aw][c], px->Ab[c][lane], xnew);
        }
        if (appends && ap.Rv) {
            __syncthreads();
            const double *Rh = ap.Rv + (size_t)h * kD * kD + r * kGroup;
            for (int e = t; e < kD * kGroup / 2; e += kThreads) {
                const int c = e >> 4, part = e & 15;
                cp_async16(&px->Ab[c][2 * part], Rh + (size_t)c * kD + 2 * part);
            }
            cp_async_commit();
            cp_async_wait<0>();
            __syncthreads();
            if (mine) {
                double y = 0.0;
#pragma unroll 16
                for (int c = 0; c < kD; c++) y = fma(px->vsd[aw][c], px->Ab[c][lane], y);
                vnew = y;
            }
        }
        // one grid per token: this CTA's share of each new token's key and
        // value ranges, met over the cluster after the barrier below
        if (NG == 1 && mine) {
            const double a = warp_min(j != 0 ? xnew : pos_inf()), bk = warp_max(j != 0 ? xnew : neg_inf());
            const double c = warp_min(vnew), d = warp_max(vnew);
            if (lane == 0) {
                px->trange[aw][0] = a;
                px->trange[aw][1] = bk;
                px->trange[aw][2] = c;
                px->trange[aw][3] = d;
            }
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
    cluster.sync();                                // every CTA's energies are ready
    for (int e = t; e < nb * kD; e += kThreads) {
        const int bi = e / kD, j = e % kD;
        const double *src = cluster.map_shared_rank(e2own, j / kGroup);
        e2s[e] = src[bi * kGroup + j % kGroup];
    }
    __syncthreads();
    // per bucket, one warp: sort the channels by (energy descending, index
    // ascending) with a bitonic network held in registers (element
    // e = 32 r + lane in register r; partners closer than 32 through
    // shuffles, the others inside the thread) -- channel 0 last (key 0; every
    // other channel's key is its energy's bit pattern + 1, and energies are
    // >= 0, so bit patterns order like values) -- then keep channel 0 and the
    // first k-1, and the per-bucket 128-bit keep masks by ballots.
    for (int bi = warp; bi < nb; bi += kThreads / 32) {
        unsigned long long key[4];
        int jj[4];
#pragma unroll
        for (int r4 = 0; r4 < 4; r4++) {
            const int j = r4 * 32 + lane;
            key[r4] = j == 0 ? 0ull : (unsigned long long)__double_as_longlong(e2s[bi * kD + j]) + 1ull;
            jj[r4] = j;
        }
#pragma unroll
        for (int size = 2; size <= kD; size <<= 1) {
#pragma unroll
            for (int stride = size >> 1; stride > 0; stride >>= 1) {
                if (stride >= 32) {
                    const int rs = stride / 32;
#pragma unroll
                    for (int ra = 0; ra < 4; ra++) {
                        if (ra & rs) continue;                   // each pair once, from its lower register
                        const int rb = ra | rs;
                        const bool up = ((ra * 32 + lane) & size) == 0;
                        const bool b_first = (key[rb] > key[ra]) || (key[rb] == key[ra] && jj[rb] < jj[ra]);
                        if (b_first == up) {
                            const unsigned long long tk = key[ra];
                            key[ra] = key[rb];
                            key[rb] = tk;
                            const int tj = jj[ra];
                            jj[ra] = jj[rb];
                            jj[rb] = tj;
                        }
                    }
                } else {
#pragma unroll
                    for (int r4 = 0; r4 < 4; r4++) {
                        const int e = r4 * 32 + lane;
                        const unsigned long long pk = __shfl_xor_sync(0xffffffffu, key[r4], stride);
                        const int pj = __shfl_xor_sync(0xffffffffu, jj[r4], stride);
                        const bool low = (e & stride) == 0, up = (e & size) == 0;
                        const bool p_first = (pk > key[r4]) || (pk == key[r4] && pj < jj[r4]);
                        // the lower element of a rising pair takes the first of the
                        // two, the upper one the second; reversed in a falling pair
                        if ((low == up) ? p_first : !p_first) {
                            key[r4] = pk;
                            jj[r4] = pj;
                        }
                    }
                }
            }
        }
#pragma unroll
        for (int r4 = 0; r4 < 4; r4++) sel[bi * kD + jj[r4]] = (jj[r4] == 0) || (r4 * 32 + lane < k - 1);
        __syncwarp();
#pragma unroll
        for (int w4 = 0; w4 < 4; w4++) {
            const unsigned m = __ballot_sync(0xffffffffu, sel[bi * kD + w4 * 32 + lane] != 0);
            if (lane == 0) mask[bi * 4 + w4] = m;
        }
    }
    __syncthreads();
    // this CTA's channels 32r..32r+31: list position = kept channels below
    for (int e = t; e < nb * kGroup; e += kThreads) {
        const int bi = e / kGroup, l = e % kGroup, c = r * kGroup + l;
        if (!sel[bi * kD + c]) continue;
        int pos = __popc(mask[bi * 4 + r] & ((1u << l) - 1u));
        for (int m = 0; m < r; m++) pos += __popc(mask[bi * 4 + m]);
        const int bk = b0 + bi;
        idx[(((size_t)b * Hkv + h) * nbk + bk) * k + pos] = c;
        for (int hl = 0; hl < g; hl++)
            qsel[((qrow0 + hl) * nbk + bk) * k + pos] = (float)qp[(bi * g + hl) * kGroup + l];
    }
    // zero-point sum of each key group (channel 0 is bf16, not in group 0),
    // kept channels ascending from 0.0: groups of 32 -- CTA r sums group r;
    // one grid per token -- CTA 0 sums all channels (reading the others' q'
    // through distributed shared memory) into entry 0, the rest are 0
    if (ng == kNG) {
        for (int e = t; e < nb * g; e += kThreads) {
            const int bi = e / g, hl = e % g;
            double s = 0.0;
            for (int l = (r == 0 ? 1 : 0); l < kGroup; l++)
                if (sel[bi * kD + r * kGroup + l]) s += qp[(bi * g + hl) * kGroup + l];
            qgsum[((qrow0 + hl) * nbk + b0 + bi) * kNG + r] = (float)s;
        }
    } else if (r == 0) {
        // all 128 channels of q' into local memory first (the rotated
        // queries are no longer needed), one parallel pass over the peers
        double *qall = sm + L.off_qr();                       // [nb][g][128]
        for (int e = t; e < nb * g * kD; e += kThreads) {
            const int row = e / kD, c = e % kD;
            qall[e] = cluster.map_shared_rank(qp, c / kGroup)[row * kGroup + c % kGroup];
        }
        __syncthreads();
        for (int e = t; e < nb * g; e += kThreads) {
            const int bi = e / g, hl = e % g;
            const double *qrow = qall + (bi * g + hl) * kD;
            double s = 0.0;
            for (int c = 1; c < kD; c++)
                if (sel[bi * kD + c]) s += qrow[c];
            float *o = qgsum + ((qrow0 + hl) * nbk + b0 + bi) * kNG;
            o[0] = (float)s;
#pragma unroll
            for (int gr = 1; gr < kNG; gr++) o[gr] = 0.f;
        }
    }
    if constexpr (APPEND) {
        // the new tokens' codes, metadata, channel 0 and protected slots (the
        // arithmetic of kvq_append); neighbouring tokens share code bytes, so
        // the rows are then merged by one thread per channel row, in order
        const bool mine = appends && aw >= 0 && aw < ap.n_new;
        uint8_t *unit = ap.pages + ((size_t)b * Hkv + h) * ap.NB * (size_t)page_bytes(2, NG);
        if (mine) {                                  // uniform over the warp
            double klo = 0.0, khi = 0.0, vlo = 0.0, vhi = 0.0;
            if constexpr (NG == 1) {
                klo = pos_inf(), khi = neg_inf(), vlo = pos_inf(), vhi = neg_inf();
#pragma unroll
                for (int rr = 0; rr < kCtas; rr++) {
                    const double *pr = cluster.map_shared_rank(&px->trange[aw][0], rr);
                    klo = fmin(klo, pr[0]);
                    khi = fmax(khi, pr[1]);
                    vlo = fmin(vlo, pr[2]);
                    vhi = fmax(vhi, pr[3]);
                }
            }
            const int pos = L0 + aw, tt = pos % kT;
            uint8_t *page = unit + (size_t)(pos / kT) * page_bytes(2, NG);
            const int mg = NG == 1 ? 0 : r;                  // metadata group
            const bool meta_writer = lane == 0 && (NG != 1 || r == 0);
            uint16_t sb, zb;
            px->kcode[aw][lane] = (uint8_t)(NG == 1 ? code_in_range<2>(xnew, klo, khi, sb, zb)
                                                    : quantize_lane<2>(xnew, j != 0, sb, zb));
            if (meta_writer)
                reinterpret_cast<uint32_t *>(page + off_kmeta(2))[meta_word(mg, tt)] = (uint32_t)sb | ((uint32_t)zb << 16);
            if (j == 0) reinterpret_cast<uint16_t *>(page + off_ch0(2))[tt] = __bfloat16_as_ushort(__double2bfloat16(xnew));
            px->vcode[aw][lane] =
                (uint8_t)(NG == 1 ? code_in_range<2>(vnew, __dmul_rn(ap.vclip, vlo), __dmul_rn(ap.vclip, vhi), sb, zb)
                                  : quantize_lane<2>(vnew, true, sb, zb, ap.vclip));
            if (meta_writer)
                reinterpret_cast<uint32_t *>(page + off_vmeta(2, NG))[meta_word(mg, tt)] = (uint32_t)sb | ((uint32_t)zb << 16);
            if (ap.n_sink + ap.n_recent > 0 && stores_slot(pos, L0 + ap.n_new, ap.n_sink, ap.n_recent)) {
                uint16_t *dst = reinterpret_cast<uint16_t *>(
                    unit_slots(ap.pages, gridDim.z, Hkv, ap.NB, 2, (size_t)b * Hkv + h, ap.n_sink + ap.n_recent, NG) +
                    (size_t)slot_of(pos, ap.n_sink, ap.n_recent) * kSlotBytes);
                dst[j] = __bfloat16_as_ushort(__double2bfloat16(xnew));
                dst[kD + j] = __bfloat16_as_ushort(__double2bfloat16(vnew));
            }
        }
        __syncthreads();
        if (appends && t >= kThreads / 2 && t < kThreads / 2 + 2 * kGroup) {
            // key row of channel 32r + (t mod 32), then the value row
            const bool val = t >= kThreads / 2 + kGroup;
            if (val || j != 0) {
                for (int i = 0; i < ap.n_new; i++) {
                    const int pos = L0 + i, tt = pos % kT;
                    const int byte = tt / 4, sh = (tt % 4) * 2;
                    uint8_t *p = unit + (size_t)(pos / kT) * page_bytes(2, NG) + (val ? off_vcodes(2) : 0) +
                                 (size_t)j * row_bytes(2) + byte;
                    const uint32_t code = val ? px->vcode[i][lane] : px->kcode[i][lane];
                    *p = (uint8_t)((*p & (uint8_t)~(3u << sh)) | (code << sh));
                }
            }
        }
    }
    cluster.sync();                                // keep e2own and qp alive until all have read them
}

template <typename Tin, bool APPEND, int NG>
cudaError_t launch_select_t(const kvq_cache &c, const void *q, int Hq, const double *Ainvt, const double *delta,
                            int k, int32_t *idx, float *qsel, float *qgsum, const StepAppend &ap, cudaStream_t st) {
    const int g = Hq / c.n_kv_heads;
    const int nbk = buckets_of(c);
    const double *rope = c.bucket > 0 ? c.rope : nullptr;
    const int nbb = rope ? std::min(nbk, std::max(1, kMaxGNbb / g)) : 1;     // buckets per cluster
    const SelLayout L{g, nbb};
    const size_t smem = APPEND ? prep_offset(L) + sizeof(PrepScratch) : L.bytes();
    // the largest layout any call can ask for (g <= 32, g * nbb <= 32 or nbb = 1)
    size_t max_smem = 0;
    for (int gg = 1; gg <= 32; gg++) {
        const SelLayout Lg{gg, std::max(1, kMaxGNbb / gg)};
        max_smem = std::max(max_smem, APPEND ? prep_offset(Lg) + sizeof(PrepScratch) : Lg.bytes());
    }
    static std::atomic<uint64_t> done{0};
    cudaError_t e = set_smem_once(select_kernel<Tin, APPEND, NG>, (int)max_smem, done);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)(kCtas * ((nbk + nbb - 1) / nbb)), (unsigned)c.n_kv_heads, (unsigned)c.batch);
    select_kernel<Tin, APPEND, NG><<<grid, kThreads, smem, st>>>(static_cast<const Tin *>(q), Ainvt, delta, Hq,
                                                                 c.n_kv_heads, g, k, idx, qsel, qgsum,
                                                                 groups_of(c), c.seq_len, rope, nbk, c.bucket, nbb,
                                                                 ap);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_select(const kvq_cache &c, const void *q, int dtype, int Hq, const double *Ainvt,
                          const double *delta, int k, int32_t *idx, float *qsel, float *qgsum, cudaStream_t st) {
    const StepAppend none{};
    return dtype == KVQ_DTYPE_F32
               ? launch_select_t<float, false, kNG>(c, q, Hq, Ainvt, delta, k, idx, qsel, qgsum, none, st)
               : launch_select_t<uint16_t, false, kNG>(c, q, Hq, Ainvt, delta, k, idx, qsel, qgsum, none, st);
}

// The first launch of a decode step (INT2, at most 4 new tokens): the
// channel choice of kvq_select_channels and the append of kvq_append, without
// the length advance; it lets the next launch on the stream start early
// (programmatic dependent launch).
cudaError_t launch_step_prep(const kvq_cache &c, const void *q, int dtype, int Hq, const void *k_new,
                             const void *v_new, int n_new, const double *A, const double *Ainvt,
                             const double *delta, int k, int32_t *idx, float *qsel, float *qgsum, cudaStream_t st) {
    const StepAppend ap{static_cast<uint8_t *>(c.pages), c.status, k_new, v_new, A, c.v_rot, value_clip(c), n_new,
                        c.capacity / kT, c.capacity, c.n_sink, c.n_recent};
    const bool one = groups_of(c) == 1;
    if (dtype == KVQ_DTYPE_F32)
        return one ? launch_select_t<float, true, 1>(c, q, Hq, Ainvt, delta, k, idx, qsel, qgsum, ap, st)
                   : launch_select_t<float, true, kNG>(c, q, Hq, Ainvt, delta, k, idx, qsel, qgsum, ap, st);
    return one ? launch_select_t<uint16_t, true, 1>(c, q, Hq, Ainvt, delta, k, idx, qsel, qgsum, ap, st)
               : launch_select_t<uint16_t, true, kNG>(c, q, Hq, Ainvt, delta, k, idx, qsel, qgsum, ap, st);
}
int step_prep_max_new() { return kPrepMaxNew; }

}  // namespace kvq
