// Decode planning (split of the context over CTAs), workspace layout and the
// choice of partial kernel; the merge is combine_kernel.
#include "kvq_internal.cuh"

#include <algorithm>

namespace kvq {

cudaError_t launch_decode_simt(const kvq_cache &c, int Hq, const int32_t *idx, const float *qsel,
                               const float *qgsum, int k, float *part_o, float2 *part_ml, int S,
                               float *out, cudaStream_t st);
cudaError_t launch_decode_mma(const kvq_cache &c, int Hq, const int32_t *idx, const float *qsel,
                              const float *qgsum, int k, float *part_o, float2 *part_ml, int S,
                              float *out, uint32_t polls, cudaStream_t st);
uint32_t default_wait_polls();
int decode_mma_splits(int units, int nblk, int num_sms, int tier);
int step_mma_max_new();
int step_mma_cluster();
cudaError_t launch_step_mma(const kvq_cache &c, int Hq, const void *q, const void *k_new, const void *v_new,
                            int dtype, int n_new, const double *A, const double *Ainvt, const double *delta,
                            int k, int32_t *idx, float *qsel, float *qgsum, float *part_o, float2 *part_ml,
                            int S, float *out, cudaStream_t st);
cudaError_t launch_decode_mma_step(const kvq_cache &c, int Hq, const int32_t *idx, const float *qsel,
                                   const float *qgsum, int k, float *part_o, float2 *part_ml, int S,
                                   float *out, int n_new, const PagePlan *plans, cudaStream_t st);
cudaError_t launch_step_prep(const kvq_cache &c, const void *q, int dtype, int Hq, const void *k_new,
                             const void *v_new, int n_new, const double *A, const double *Ainvt,
                             const double *delta, int k, int32_t *idx, float *qsel, float *qgsum, PagePlan *plans,
                             bool append_here, cudaStream_t st);
cudaError_t launch_step_append(const kvq_cache &c, const void *K, const void *V, int dtype, int n_new,
                               const double *A, cudaStream_t st);
int step_prep_max_new();

// The tensor-core kernel covers INT2 codes with 4 query heads per KV head;
// other shapes use the CUDA-core kernel.
static bool use_mma(const kvq_cache &c, int Hq) { return c.bits == 2 && Hq == 4 * c.n_kv_heads; }

// Splits per (sequence, KV head): enough CTAs to fill the SMs (the
// tensor-core plan: decode_mma_splits), at least two pages per split for the
// CUDA-core kernel, and at most kMaxSplits (which bounds the workspace).
constexpr int kMaxSplits = 256;

int decode_splits(const kvq_cache &c, int Hq, int k, int num_sms) {
    (void)k;
    const int units = c.batch * c.n_kv_heads;
    const int nblk = c.capacity / kT;
    const int tier = tier_ctas(c);                 // extra splits that read the protected tier
    int S;
    if (use_mma(c, Hq)) {
        S = decode_mma_splits(units, nblk, num_sms, tier);
    } else {
        S = (4 * num_sms + units - 1) / units;
        const int max_s = (nblk + 1) / 2 > 0 ? (nblk + 1) / 2 : 1;
        if (S > max_s) S = max_s;
        if (S < 1) S = 1;
        S += tier;
    }
    if (S > kMaxSplits) S = kMaxSplits;
    return S;
}

// The one-launch step (tensor-core shape, no RoPE buckets) runs as clusters
// of consecutive splits: its page splits are the decode's rounded down to
// the cluster size (at least one cluster), plus the tier's.
static bool fused_step(const kvq_cache &c, int Hq, int n_new) {
    return use_mma(c, Hq) && c.bucket == 0 && n_new <= step_mma_max_new();
}
static int step_splits(const kvq_cache &c, int S) {
    const int tier = tier_ctas(c), cl = step_mma_cluster();
    int pages = S - tier;
    pages -= pages % cl;
    return (pages < cl ? cl : pages) + tier;
}

// Workspace: the split partials (o, then (m, l)) and, for the tensor-core
// shape, a decode step's page plans (one per sequence, KV head and RoPE
// bucket) after them at a 16-byte boundary; for a step, partials of the
// larger of the decode's and the one-launch step's split counts.
static size_t partials_bytes(const kvq_cache &c, int Hq, int S) {
    return ((size_t)c.batch * Hq * S * (kD * sizeof(float) + sizeof(float2)) + 15) & ~(size_t)15;
}
size_t decode_ws_bytes(const kvq_cache &c, int Hq, int S, bool step) {
    if (!step) return partials_bytes(c, Hq, S);
    size_t n = partials_bytes(c, Hq, use_mma(c, Hq) ? std::max(S, step_splits(c, S)) : S);
    if (use_mma(c, Hq)) n += (size_t)c.batch * c.n_kv_heads * buckets_of(c) * sizeof(PagePlan);
    return n;
}

// polls < 0: the tensor-core kernel's default bound on each wait for a
// staged page; any other value replaces it (0: give up unless the page has
// already landed -- the test path for the give-up).
cudaError_t launch_decode(const kvq_cache &c, int Hq, const int32_t *idx, const float *qsel,
                          const float *qgsum, int k, float *out, void *ws, int S, cudaStream_t st,
                          long long polls) {
    float *part_o = static_cast<float *>(ws);
    float2 *part_ml = reinterpret_cast<float2 *>(part_o + (size_t)c.batch * Hq * S * kD);
    // one launch: the last CTA of each (sequence, KV head) merges the splits
    return use_mma(c, Hq) ? launch_decode_mma(c, Hq, idx, qsel, qgsum, k, part_o, part_ml, S, out,
                                              polls < 0 ? default_wait_polls() : (uint32_t)polls, st)
                          : launch_decode_simt(c, Hq, idx, qsel, qgsum, k, part_o, part_ml, S, out, st);
}
bool decode_uses_mma(const kvq_cache &c, int Hq) { return use_mma(c, Hq); }

// One decode step.  The tensor-core shape with at most 4 new tokens runs as
// one fused launch without RoPE buckets.  With buckets it is a chain of
// programmatic dependent launches: the append of the new tokens (without the
// length advance), the channel choice of every bucket with the page plans
// (which starts while the append runs and waits for it before it exits), and
// the decode, which waits for the choice and advances the length.  Anything
// else runs as the three calls.
cudaError_t launch_decode_step(const kvq_cache &c, int Hq, const void *q, const void *k_new,
                               const void *v_new, int dtype, int n_new, const double *A,
                               const double *Ainvt, const double *delta, int k, int32_t *idx, float *qsel,
                               float *qgsum, float *out, void *ws, int S, cudaStream_t st) {
    if (fused_step(c, Hq, n_new)) {
        const int Ss = step_splits(c, S);
        float *part_o = static_cast<float *>(ws);
        float2 *part_ml = reinterpret_cast<float2 *>(part_o + (size_t)c.batch * Hq * Ss * kD);
        return launch_step_mma(c, Hq, q, k_new, v_new, dtype, n_new, A, Ainvt, delta, k, idx, qsel, qgsum, part_o,
                               part_ml, Ss, out, st);
    }
    if (use_mma(c, Hq) && n_new <= step_prep_max_new()) {
        float *part_o = static_cast<float *>(ws);
        float2 *part_ml = reinterpret_cast<float2 *>(part_o + (size_t)c.batch * Hq * S * kD);
        PagePlan *plans = reinterpret_cast<PagePlan *>(static_cast<uint8_t *>(ws) + partials_bytes(c, Hq, S));
        cudaError_t e = cudaSuccess;
        if (n_new > 0) e = launch_step_append(c, k_new, v_new, dtype, n_new, A, st);
        if (e == cudaSuccess)
            e = launch_step_prep(c, q, dtype, Hq, k_new, v_new, n_new, A, Ainvt, delta, k, idx, qsel, qgsum, plans,
                                 n_new == 0, st);
        if (e == cudaSuccess)
            e = launch_decode_mma_step(c, Hq, idx, qsel, qgsum, k, part_o, part_ml, S, out, n_new, plans, st);
        return e;
    }
    cudaError_t e = cudaSuccess;
    if (n_new > 0) e = launch_append(c, k_new, v_new, dtype, n_new, A, st);
    if (e == cudaSuccess) e = launch_select(c, q, dtype, Hq, Ainvt, delta, k, idx, qsel, qgsum, st);
    if (e == cudaSuccess) e = launch_decode(c, Hq, idx, qsel, qgsum, k, out, ws, S, st);
    return e;
}

}  // namespace kvq
