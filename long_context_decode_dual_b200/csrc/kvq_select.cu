// kvq_select_channels: query transform and top-k channel choice.
//
// "Dual-QK: Sharp Queries and Flat Keys for Prunable 2-bit KV Caches":
//   §3.1 the query is multiplied by the inverse transpose of the key
//        transform, so transformed scores equal the original ones;
//   §3.2 Eq. 4: channel energy pooled over the query heads sharing a KV head,
//        e_j^2 = sum_h q'_{h,j}^2, one mask per KV head, chosen per query.
// Channel 0 is always kept; ties go to the lower channel index.
//
// One CTA = one (sequence, KV head), 512 threads.  A^{-T} of the head is
// staged in shared memory with one cp.async burst, then thread (slot, j) runs
// the fixed-order fp64 fma chains q'[h][j] for heads h = slot, slot+4, ....  The selection is
// exact and order-free: each candidate counts the channels that beat it
// (rank, split four ways), then a ballot prefix sum writes the kept channels
// in ascending order.
#include "kvq_internal.cuh"

namespace kvq {
namespace {

constexpr int kThreads = 512;

template <typename Tin>
__global__ void __launch_bounds__(kThreads)
select_kernel(const Tin *__restrict__ q, const double *__restrict__ Ainvt, int Hq, int Hkv, int g,
              int k, int32_t *__restrict__ idx, float *__restrict__ qsel,
              float *__restrict__ qgsum) {
    extern __shared__ __align__(16) double sm[];   // Ainvt[128][128], qin[g][128], qp[g][128]
    double *As = sm;
    double *qin = sm + kD * kD;
    double *qp = qin + (size_t)g * kD;
    __shared__ double e2s[kD];
    __shared__ int rank_part[4][kD];
    __shared__ int sel_s[kD];
    __shared__ int warp_cnt[4];

    const int h = blockIdx.x, b = blockIdx.y, t = threadIdx.x;
    const int j = t & (kD - 1), slot = t >> 7;
    const size_t qrow0 = (size_t)b * Hq + (size_t)h * g;

    // A^{-T} of this KV head in one cp.async burst
    const double *Ai = Ainvt + (size_t)h * kD * kD;
    for (int e = t; e < kD * kD / 2; e += kThreads) cp_async16(As + 2 * e, Ai + 2 * e);
    cp_async_commit();
    for (int e = t; e < g * kD; e += kThreads) qin[e] = in_to_double(q[qrow0 * kD + e]);
    cp_async_wait<0>();
    __syncthreads();

    // q'[hl][j] = sum_c q[hl][c] Ainvt[c][j], fma chain c = 0..127 from 0.0
    for (int hl = slot; hl < g; hl += 4) {
        double acc = 0.0;
#pragma unroll 16
        for (int c = 0; c < kD; c++) acc = fma(qin[hl * kD + c], As[c * kD + j], acc);
        qp[hl * kD + j] = acc;
    }
    __syncthreads();
    // e_j^2, fma chain over heads ascending from 0.0
    if (t < kD) {
        double e = 0.0;
        for (int hl = 0; hl < g; hl++) e = fma(qp[hl * kD + j], qp[hl * kD + j], e);
        e2s[j] = e;
    }
    __syncthreads();
    // rank of candidate j >= 1 among channels 1..127, counted in four parts
    {
        const double e = e2s[j];
        int r = 0;
        const int i0 = 1 + 32 * slot, i1 = min(kD, i0 + 32);
        for (int i = i0; i < i1; i++) {
            const double ei = e2s[i];
            r += (ei > e) || (ei == e && i < j);
        }
        rank_part[slot][j] = r;
    }
    __syncthreads();
    if (t < kD) {
        const int lane = t & 31, warp = t >> 5;
        const bool sel = (j == 0) ||
                         (rank_part[0][j] + rank_part[1][j] + rank_part[2][j] + rank_part[3][j] < k - 1);
        sel_s[j] = sel;
        const unsigned ballot = __ballot_sync(0xffffffffu, sel);
        if (lane == 0) warp_cnt[warp] = __popc(ballot);
        __syncwarp();
        // (warp_cnt of the other warps is read after the barrier below)
        rank_part[0][j] = sel ? (int)__popc(ballot & ((1u << lane) - 1u)) : -1;
    }
    __syncthreads();
    if (t < kD) {
        int pos = rank_part[0][j];
        if (pos >= 0) {
            for (int w = 0; w < (t >> 5); w++) pos += warp_cnt[w];
            idx[((size_t)b * Hkv + h) * k + pos] = j;
            for (int hl = 0; hl < g; hl++) qsel[(qrow0 + hl) * k + pos] = (float)qp[hl * kD + j];
        }
    }
    // zero-point sums per key group (channel 0 is bf16, not in group 0)
    for (int u = t; u < g * kNG; u += kThreads) {
        const int hl = u / kNG, gr = u % kNG;
        double s = 0.0;
        for (int c = (gr == 0 ? 1 : gr * kGroup); c < (gr + 1) * kGroup; c++)
            if (sel_s[c]) s += qp[hl * kD + c];
        qgsum[(qrow0 + hl) * kNG + gr] = (float)s;
    }
}

}  // namespace

cudaError_t launch_select(const kvq_cache &c, const void *q, int dtype, int Hq, const double *Ainvt,
                          int k, int32_t *idx, float *qsel, float *qgsum, cudaStream_t st) {
    const int g = Hq / c.n_kv_heads;
    const size_t smem = (size_t)(kD * kD + 2 * g * kD) * sizeof(double);
    constexpr int kMaxSmem = (kD * kD + 2 * 32 * kD) * (int)sizeof(double);      // g <= 32
    static std::atomic<uint64_t> done_f32{0}, done_bf16{0};
    dim3 grid((unsigned)c.n_kv_heads, (unsigned)c.batch);
    cudaError_t e;
    if (dtype == KVQ_DTYPE_F32) {
        e = set_smem_once(select_kernel<float>, kMaxSmem, done_f32);
        if (e != cudaSuccess) return e;
        select_kernel<float><<<grid, kThreads, smem, st>>>(static_cast<const float *>(q), Ainvt, Hq,
                                                           c.n_kv_heads, g, k, idx, qsel, qgsum);
    } else {
        e = set_smem_once(select_kernel<uint16_t>, kMaxSmem, done_bf16);
        if (e != cudaSuccess) return e;
        select_kernel<uint16_t><<<grid, kThreads, smem, st>>>(static_cast<const uint16_t *>(q), Ainvt, Hq,
                                                              c.n_kv_heads, g, k, idx, qsel, qgsum);
    }
    return cudaGetLastError();
}

}  // namespace kvq
