// kvq_select_channels: query transform and top-k channel choice.
//
// "Dual-QK: Sharp Queries and Flat Keys for Prunable 2-bit KV Caches":
//   §3.1 the query is multiplied by the inverse transpose of the key
//        transform, so transformed scores equal the original ones;
//   §3.2 Eq. 4: channel energy pooled over the query heads sharing a KV head,
//        e_j^2 = sum_h q'_{h,j}^2, one mask per KV head, chosen per query;
//   §3.3, App. C.2: with a diagonal refinement D folded into the transforms
//        the energies are those of the base queries, q'_{h,j} / delta_j.
// Channel 0 is always kept; ties go to the lower channel index.
//
// With bucket-relative RoPE (§3.4) the grid has one cluster per bucket too:
// the cluster of bucket b first moves the query into b's frame (its anchor's
// rotary rotation removed) and writes entry b of the outputs; buckets past
// the sequence's length (other than bucket 0) do nothing.
//
// One thread-block cluster of four CTAs = one (sequence, KV head); CTA r owns
// channels 32r..32r+31 (key group r).  It stages its 32 columns of A^{-T}
// (32 KB) with one cp.async burst and runs the fixed-order fp64 fma chains
// q'[h][j] of its channels, then their pooled energies.  After a cluster
// barrier every CTA reads the four energy blocks through distributed shared
// memory and makes the same exact, order-free choice (each candidate counts
// the channels that beat it), so no CTA waits for another's decision; each
// writes the outputs of its own channels: their list positions (a ballot
// prefix sum over the 128 flags), q' in fp32 and its group's zero-point sum.
#include "kvq_internal.cuh"

#include <cooperative_groups.h>

namespace kvq {
namespace {

namespace cg = cooperative_groups;

constexpr int kThreads = 256;
constexpr int kCtas = kNG;                 // CTAs per cluster, one per key group

template <typename Tin>
__global__ void __cluster_dims__(kCtas, 1, 1) __launch_bounds__(kThreads)
select_kernel(const Tin *__restrict__ q, const double *__restrict__ Ainvt, const double *__restrict__ delta,
              int Hq, int Hkv, int g, int k, int32_t *__restrict__ idx, float *__restrict__ qsel,
              float *__restrict__ qgsum, int ng, const int32_t *__restrict__ seq_len,
              const double *__restrict__ rope, int nbk, int w) {
    extern __shared__ __align__(16) double sm[];   // As[128][32], qin[g][128], qp[g][32]
    double *As = sm;
    double *qin = sm + kD * kGroup;
    double *qp = qin + (size_t)g * kD;
    __shared__ double e2own[kGroup];
    __shared__ double e2s[kD];
    __shared__ int rank_part[2][kD];
    __shared__ int sel_s[kD];
    __shared__ int warp_cnt[4];

    cg::cluster_group cluster = cg::this_cluster();
    const int r = (int)cluster.block_rank();       // = blockIdx.x % 4
    const int bk = blockIdx.x / kCtas;              // RoPE bucket (0 without buckets)
    const int h = blockIdx.y, b = blockIdx.z, t = threadIdx.x;
    const int lane = t & 31, warp = t >> 5;
    const size_t qrow0 = (size_t)b * Hq + (size_t)h * g;
    if (bk > 0 && (size_t)bk * w >= (size_t)max(seq_len[b], 0)) return;   // the whole cluster

    // columns 32r..32r+31 of A^{-T} for this KV head: 128 rows of 256 bytes
    const double *Ai = Ainvt + (size_t)h * kD * kD + r * kGroup;
    for (int e = t; e < kD * kGroup / 2; e += kThreads) {
        const int c = e >> 4, part = e & 15;
        cp_async16(As + c * kGroup + 2 * part, Ai + (size_t)c * kD + 2 * part);
    }
    cp_async_commit();
    for (int e = t; e < g * kD; e += kThreads) qin[e] = in_to_double(q[qrow0 * kD + e]);
    cp_async_wait<0>();
    __syncthreads();
    if (rope) {
        // q T_b: channel pairs (i, i + 64) rotated back by the anchor's angle
        const double2 *cs = reinterpret_cast<const double2 *>(rope) + (size_t)bk * (kD / 2);
        for (int e = t; e < g * (kD / 2); e += kThreads) {
            const int hl = e / (kD / 2), i = e % (kD / 2);
            rope_unanchor_pair(qin[hl * kD + i], qin[hl * kD + i + kD / 2], __ldg(cs + i));
        }
        __syncthreads();
    }

    // q'[hl][j] = sum_c q[hl][c] Ainvt[c][j], fma chain c = 0..127 from 0.0
    for (int hl = warp; hl < g; hl += kThreads / 32) {
        double acc = 0.0;
#pragma unroll 16
        for (int c = 0; c < kD; c++) acc = fma(qin[hl * kD + c], As[c * kGroup + lane], acc);
        qp[hl * kGroup + lane] = acc;
    }
    __syncthreads();
    // e_j^2, fma chain over heads ascending from 0.0; with a diagonal
    // refinement D, of the base queries q'_{h,j} / delta_j
    if (t < kGroup) {
        const double dj = delta ? delta[(size_t)h * kD + r * kGroup + t] : 1.0;
        double e = 0.0;
        for (int hl = 0; hl < g; hl++) {
            const double u = delta ? qp[hl * kGroup + t] / dj : qp[hl * kGroup + t];
            e = fma(u, u, e);
        }
        e2own[t] = e;
    }
    cluster.sync();                                // every CTA's energies are ready
    if (t < kD) {
        const double *src = cluster.map_shared_rank(e2own, t / kGroup);
        e2s[t] = src[t % kGroup];
    }
    __syncthreads();
    // rank of candidate j >= 1 among channels 1..127, counted in two halves
    {
        const int j = t & (kD - 1), part = t >> 7;
        // energies are >= 0, so their bit patterns order like their values
        const unsigned long long e = __double_as_longlong(e2s[j]);
        int rk = 0;
        const int i0 = part == 0 ? 1 : 64, i1 = part == 0 ? 64 : kD;
#pragma unroll 4
        for (int i = i0; i < i1; i++) {
            const unsigned long long ei = __double_as_longlong(e2s[i]);
            rk += (ei > e) || (ei == e && i < j);
        }
        rank_part[part][j] = rk;
    }
    __syncthreads();
    int pos = -1;
    if (t < kD) {
        const bool sel = (t == 0) || (rank_part[0][t] + rank_part[1][t] < k - 1);
        sel_s[t] = sel;
        const unsigned ballot = __ballot_sync(0xffffffffu, sel);
        if (lane == 0) warp_cnt[warp] = __popc(ballot);
        if (sel) pos = (int)__popc(ballot & ((1u << lane) - 1u));
    }
    __syncthreads();
    // this CTA's channels are t = 32r..32r+31 (warp r)
    if (warp == r && pos >= 0) {
        for (int w = 0; w < r; w++) pos += warp_cnt[w];
        idx[(((size_t)b * Hkv + h) * nbk + bk) * k + pos] = t;
        for (int hl = 0; hl < g; hl++) qsel[((qrow0 + hl) * nbk + bk) * k + pos] = (float)qp[hl * kGroup + lane];
    }
    // zero-point sum of each key group (channel 0 is bf16, not in group 0),
    // kept channels ascending from 0.0: groups of 32 -- CTA r sums group r;
    // one grid per token -- CTA 0 sums all channels (reading the others' q'
    // through distributed shared memory) into entry 0, the rest are 0
    if (ng == kNG) {
        for (int hl = t; hl < g; hl += kThreads) {
            double s = 0.0;
            for (int c = (r == 0 ? 1 : 0); c < kGroup; c++)
                if (sel_s[r * kGroup + c]) s += qp[hl * kGroup + c];
            qgsum[((qrow0 + hl) * nbk + bk) * kNG + r] = (float)s;
        }
    } else if (r == 0) {
        const double *pq[kCtas];
#pragma unroll
        for (int rr = 0; rr < kCtas; rr++) pq[rr] = cluster.map_shared_rank(qp, rr);
        for (int hl = t; hl < g; hl += kThreads) {
            double s = 0.0;
            for (int c = 1; c < kD; c++)
                if (sel_s[c]) s += pq[c / kGroup][hl * kGroup + c % kGroup];
            qgsum[((qrow0 + hl) * nbk + bk) * kNG] = (float)s;
#pragma unroll
            for (int gr = 1; gr < kNG; gr++) qgsum[((qrow0 + hl) * nbk + bk) * kNG + gr] = 0.f;
        }
    }
    cluster.sync();                                // keep e2own alive until all have read it
}

}  // namespace

cudaError_t launch_select(const kvq_cache &c, const void *q, int dtype, int Hq, const double *Ainvt,
                          const double *delta, int k, int32_t *idx, float *qsel, float *qgsum, cudaStream_t st) {
    const int g = Hq / c.n_kv_heads;
    const size_t smem = (size_t)(kD * kGroup + g * kD + g * kGroup) * sizeof(double);
    constexpr int kMaxSmem = (kD * kGroup + 32 * kD + 32 * kGroup) * (int)sizeof(double);   // g <= 32
    static std::atomic<uint64_t> done_f32{0}, done_bf16{0};
    const int nbk = buckets_of(c);
    dim3 grid((unsigned)(kCtas * nbk), (unsigned)c.n_kv_heads, (unsigned)c.batch);
    const double *rope = c.bucket > 0 ? c.rope : nullptr;
    cudaError_t e;
    if (dtype == KVQ_DTYPE_F32) {
        e = set_smem_once(select_kernel<float>, kMaxSmem, done_f32);
        if (e != cudaSuccess) return e;
        select_kernel<float><<<grid, kThreads, smem, st>>>(static_cast<const float *>(q), Ainvt, delta, Hq,
                                                           c.n_kv_heads, g, k, idx, qsel, qgsum, groups_of(c),
                                                           c.seq_len, rope, nbk, c.bucket);
    } else {
        e = set_smem_once(select_kernel<uint16_t>, kMaxSmem, done_bf16);
        if (e != cudaSuccess) return e;
        select_kernel<uint16_t><<<grid, kThreads, smem, st>>>(static_cast<const uint16_t *>(q), Ainvt, delta, Hq,
                                                              c.n_kv_heads, g, k, idx, qsel, qgsum, groups_of(c),
                                                              c.seq_len, rope, nbk, c.bucket);
    }
    return cudaGetLastError();
}

}  // namespace kvq
