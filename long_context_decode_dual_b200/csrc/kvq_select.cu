// kvq_select_channels: query transform and top-k channel choice.
//
// "Dual-QK: Sharp Queries and Flat Keys for Prunable 2-bit KV Caches":
//   §3.1 the query is multiplied by the inverse transpose of the key
//        transform, so transformed scores equal the original ones;
//   §3.2 Eq. 4: channel energy pooled over the query heads sharing a KV head,
//        e_j^2 = sum_h q'_{h,j}^2, one mask per KV head, chosen per query.
// Channel 0 is always kept; ties go to the lower channel index.
//
// One CTA = one (sequence, KV head); thread j owns channel j.  The selection
// is exact: each candidate counts how many channels beat it (rank), which is
// order-free, then a ballot prefix sum writes the kept channels ascending.
#include "kvq_internal.cuh"

namespace kvq {
namespace {

constexpr int kMaxG = 32;

template <typename Tin>
__global__ void __launch_bounds__(128)
select_kernel(const Tin *__restrict__ q, const double *__restrict__ Ainvt, int Hq, int Hkv, int g,
              int k, int32_t *__restrict__ idx, float *__restrict__ qsel,
              float *__restrict__ qgsum) {
    extern __shared__ double sm[];          // qin[g][128], qp[g][128]
    double *qin = sm;
    double *qp = sm + (size_t)g * kD;
    __shared__ double e2s[kD];
    __shared__ int sel_s[kD];
    __shared__ int warp_cnt[4];

    const int h = blockIdx.x, b = blockIdx.y, j = threadIdx.x;
    const int lane = j & 31, warp = j >> 5;
    const size_t qrow0 = (size_t)b * Hq + (size_t)h * g;

    for (int e = j; e < g * kD; e += blockDim.x) qin[e] = in_to_double(q[qrow0 * kD + e]);
    __syncthreads();

    // q'[hl][j] = sum_c q[hl][c] Ainvt[c][j], fma chain c = 0..127 from 0.0
    const double *Ai = Ainvt + (size_t)h * kD * kD + j;
    for (int hl = 0; hl < g; hl++) {
        double acc = 0.0;
#pragma unroll 8
        for (int c = 0; c < kD; c++) acc = fma(qin[hl * kD + c], __ldg(Ai + (size_t)c * kD), acc);
        qp[hl * kD + j] = acc;
    }
    // e_j^2, fma chain over heads ascending from 0.0
    double e = 0.0;
    for (int hl = 0; hl < g; hl++) e = fma(qp[hl * kD + j], qp[hl * kD + j], e);
    e2s[j] = e;
    __syncthreads();

    bool sel;
    if (j == 0) {
        sel = true;
    } else {
        int rank = 0;
        for (int i = 1; i < kD; i++) {
            const double ei = e2s[i];
            rank += (ei > e) || (ei == e && i < j);
        }
        sel = rank < k - 1;
    }
    sel_s[j] = sel;
    const unsigned ballot = __ballot_sync(0xffffffffu, sel);
    if (lane == 0) warp_cnt[warp] = __popc(ballot);
    __syncthreads();
    int pos = __popc(ballot & ((1u << lane) - 1u));
    for (int w = 0; w < warp; w++) pos += warp_cnt[w];

    if (sel) {
        idx[((size_t)b * Hkv + h) * k + pos] = j;
        for (int hl = 0; hl < g; hl++) qsel[(qrow0 + hl) * k + pos] = (float)qp[hl * kD + j];
    }
    // zero-point sums per key group (channel 0 is bf16, not in group 0)
    for (int t = j; t < g * kNG; t += blockDim.x) {
        const int hl = t / kNG, gr = t % kNG;
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
    const size_t smem = (size_t)2 * g * kD * sizeof(double);
    dim3 grid((unsigned)c.n_kv_heads, (unsigned)c.batch);
    if (dtype == KVQ_DTYPE_F32) {
        cudaFuncSetAttribute(select_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        select_kernel<float><<<grid, 128, smem, st>>>(static_cast<const float *>(q), Ainvt, Hq,
                                                      c.n_kv_heads, g, k, idx, qsel, qgsum);
    } else {
        cudaFuncSetAttribute(select_kernel<uint16_t>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        select_kernel<uint16_t><<<grid, 128, smem, st>>>(static_cast<const uint16_t *>(q), Ainvt, Hq,
                                                         c.n_kv_heads, g, k, idx, qsel, qgsum);
    }
    return cudaGetLastError();
}

static_assert(kMaxG * 2 * kD * sizeof(double) <= 227 * 1024, "select smem");

}  // namespace kvq
