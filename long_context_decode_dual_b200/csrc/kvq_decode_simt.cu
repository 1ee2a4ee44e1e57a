// Channel-skipping decode attention, CUDA-core variant (any GQA group size
// up to 8 query heads per KV head, INT2 or INT4 codes), and the split merge.
//
// "Dual-QK: Sharp Queries and Flat Keys for Prunable 2-bit KV Caches":
//   §3.2 scores use only the retained key channels and keep the 1/sqrt(d)
//        normalisation of the full dimension;
//   §3.3 the decode kernel copies asynchronously only the 32-byte key rows
//        selected by the shared query mask; values and metadata are read in
//        full;
//   §3.4 scores from the whole cache share one softmax, followed by value
//        aggregation.
// The context is split over CTAs (flash-decoding); each keeps a running max,
// sum and output per query head, merged exactly by combine_kernel.
//
// One CTA = one (sequence, KV head, split), 128 threads.  Per 128-token page:
// the selected key rows and the fixed part (value codes, channel 0, key and
// value metadata) are staged in shared memory with cp.async (double
// buffered); thread t scores token t, then thread c accumulates value
// channel c.  The dot product is factored per key group so that codes are
// multiplied by the query first and the group's scale and zero-point are
// applied once:  q.k_hat = s_g * sum_{c in S_g} q_c code_c + z_g * sum_{c in S_g} q_c.
#include "kvq_internal.cuh"

namespace kvq {
namespace {

template <int G>
struct SimtSmem {
    // byte offsets of the small arrays after the two stages
    static constexpr int q_bytes = kD * G * 4;      // qsel [i][G]
    static constexpr int qg_bytes = kNG * G * 4;    // qgsum [gr][G]
    static constexpr int idx_bytes = kD * 4;
    static constexpr int p_bytes = kD * G * 4;      // p [t][G]
    static constexpr int red_bytes = 4 * G * 4;
    static constexpr int extra = q_bytes + qg_bytes + idx_bytes + p_bytes + red_bytes + 32;
};

__device__ __forceinline__ float warp_max_f(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ float h2f_lo(uint32_t w) { return __half2float(__ushort_as_half((uint16_t)(w & 0xffffu))); }
__device__ __forceinline__ float h2f_hi(uint32_t w) { return __half2float(__ushort_as_half((uint16_t)(w >> 16))); }

template <int BITS, int G, int NG>
__global__ void __launch_bounds__(128)
decode_simt_kernel(const uint8_t *__restrict__ pages, const int32_t *__restrict__ seq_len, int Hkv,
                   int NB, int Hq, const int32_t *__restrict__ idx, const float *__restrict__ qsel,
                   const float *__restrict__ qgsum, int k, float *__restrict__ part_o,
                   float2 *__restrict__ part_ml, int S, float *__restrict__ out,
                   uint32_t *__restrict__ counters, uint32_t *__restrict__ status, int n_sink, int n_recent,
                   int stage_area, const double *__restrict__ v_rot, int nbk, int w_pages) {
    constexpr int R = row_bytes(BITS);
    constexpr int FIX = fixed_bytes(BITS, NG);
    constexpr int GS = kD / NG;                       // channels per quantization group
    constexpr int PER = 8 / BITS;
    constexpr uint32_t CMASK = (1u << BITS) - 1u;
    using SM = SimtSmem<G>;

    extern __shared__ __align__(16) uint8_t smem[];
    const int s = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int ksel = k - 1;
    const int stage_bytes = ksel * R + FIX;
    uint8_t *stage[2] = {smem, smem + stage_bytes};
    float *sq = reinterpret_cast<float *>(smem + stage_area);     // stage_area >= 2 * stage_bytes
    float *sqg = sq + kD * G;
    int *sidx = reinterpret_cast<int *>(sqg + kNG * G);
    float *sp = reinterpret_cast<float *>(sidx + kD);
    float *sred = sp + kD * G;
    int *sgs = reinterpret_cast<int *>(sred + 4 * G);

    const size_t unit = (size_t)b * Hkv + h;
    const size_t qrow0 = (size_t)b * Hq + (size_t)h * G;
    // channel choice of bucket bk (0 without RoPE buckets) into shared memory.
    // The list must be channel 0 followed by ascending channels in 1..127;
    // another list is clamped into the page and raises KVQ_DEV_INDEX.
    auto load_sel = [&](int bk) {
        const int32_t *sel = idx + (unit * nbk + bk) * k;
        bool bad = false;
        for (int i = tid; i < k; i += 128) {
            const int c = sel[i];
            bad |= (i == 0) ? c != 0 : (c <= sel[i - 1] || c > kD - 1);
            sidx[i] = min(max(c, 0), kD - 1);
        }
        for (int e = tid; e < G * k; e += 128) {
            const int hl = e / k, i = e % k;
            sq[i * G + hl] = qsel[((qrow0 + hl) * nbk + bk) * k + i];
        }
        if (tid < G * kNG) {
            const int hl = tid / kNG, gr = tid % kNG;
            sqg[gr * G + hl] = qgsum[((qrow0 + hl) * nbk + bk) * kNG + gr];
        }
        if (__syncthreads_or(bad) && tid == 0) atomicOr(status, (uint32_t)KVQ_DEV_INDEX);
        if (tid == 0) {
            // selected list positions 1..k-1 hold channels >= 1 ascending; group
            // gr spans positions [sgs[gr], sgs[gr+1])
            int i = 1;
            for (int gr = 0; gr < NG; gr++) {
                sgs[gr] = i;
                while (i < k && sidx[i] < (gr + 1) * GS) i++;
            }
            sgs[NG] = k;
        }
        __syncthreads();
    };

    // a caller-owned length outside [0, capacity] is clamped, never followed
    const int len = min(max(seq_len[b], 0), NB * kT);
    // with a protected tier the last two splits read its BF16 slots; the
    // pages cover the coded tokens [lo, hi)
    const int NPt = n_sink + n_recent;
    const int S_pages = S - (NPt > 0 ? 2 : 0);
    if (s >= S_pages) {
        const int per = (NPt + 1) / 2;
        const int slot0 = min(NPt, (s - S_pages) * per), slot1 = min(NPt, slot0 + per);
        const uint8_t *slots = unit_slots(const_cast<uint8_t *>(pages), gridDim.z, Hkv, NB, BITS, unit, NPt, NG);
        if (w_pages > 0) {
            tier_partial<G, 128>(slots, len, n_sink, n_recent, slot0, slot1,
                                 TierQBuckets{qsel, idx + unit * nbk * k, k, nbk, w_pages * kT, qrow0}, k, part_o,
                                 part_ml, qrow0, S, s, reinterpret_cast<float *>(smem));
        } else {
            load_sel(0);
            tier_partial<G, 128>(slots, len, n_sink, n_recent, slot0, slot1, TierQShared{sq, 1, G, sidx}, k, part_o,
                                 part_ml, qrow0, S, s, reinterpret_cast<float *>(smem));
        }
        merge_unit_if_last<G, 128>(part_o, part_ml, S, qrow0, out, counters + unit, reinterpret_cast<float *>(smem),
                                   v_rot ? v_rot + (size_t)h * kD * kD : nullptr);
        return;
    }
    const Tier tr = tier_of(len, n_sink, n_recent);
    const int lo = tr.sink_end, hi = tr.recent_start;
    const int nblk = (hi + kT - 1) / kT;
    const int bps = (nblk + S_pages - 1) / S_pages;
    const int blk0 = s * bps;
    const int blk1 = min(nblk, blk0 + bps);

    auto load = [&](uint8_t *dst, int blk) {
        const uint8_t *pg = pages + (unit * NB + (size_t)blk) * page_bytes(BITS, NG);
        constexpr int CPR = R / 16;
        for (int e = tid; e < ksel * CPR; e += 128) {
            const int i = e / CPR, part = e % CPR;
            cp_async16(dst + i * R + part * 16, pg + (size_t)sidx[i + 1] * R + part * 16);
        }
        for (int e = tid; e < FIX / 16; e += 128)
            cp_async16(dst + ksel * R + e * 16, pg + off_vcodes(BITS) + e * 16);
        cp_async_commit();
    };

    float m_run[G], l_run[G], o_acc[G];
#pragma unroll
    for (int hl = 0; hl < G; hl++) {
        m_run[hl] = -INFINITY;
        l_run[hl] = 0.f;
        o_acc[hl] = 0.f;
    }

    // pages [blk0, blk1) as segments, one per RoPE bucket (one segment
    // without buckets); the softmax state runs on across segments
    if (w_pages == 0) load_sel(0);
    for (int seg0 = blk0; seg0 < blk1;) {
    const int seg1 = w_pages > 0 ? min(blk1, (seg0 / w_pages + 1) * w_pages) : blk1;
    if (w_pages > 0) load_sel(seg0 / w_pages);      // the last page's barrier has passed
    load(stage[0], seg0);
    for (int blk = seg0; blk < seg1; blk++) {
        uint8_t *cur = stage[(blk - seg0) & 1];
        if (blk + 1 < seg1) {
            load(stage[(blk - seg0 + 1) & 1], blk + 1);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();

        const uint8_t *krows = cur;
        const uint8_t *vcodes = cur + ksel * R;
        const uint16_t *ch0 = reinterpret_cast<const uint16_t *>(vcodes + 128 * R);
        const uint32_t *kmeta = reinterpret_cast<const uint32_t *>(vcodes + 128 * R + 256);
        const uint32_t *vmeta = kmeta + NG * kT;

        // ---- scores: thread t = token t of the page
        {
            const int t = tid;
            const bool valid = blk * kT + t >= lo && blk * kT + t < hi;
            float sc[G];
            const float c0 = __uint_as_float(((uint32_t)ch0[t]) << 16);
#pragma unroll
            for (int hl = 0; hl < G; hl++) sc[hl] = sq[hl] * c0;
            const int boff = t / PER, sh = (t % PER) * BITS;
#pragma unroll
            for (int gr = 0; gr < NG; gr++) {
                float d[G];
#pragma unroll
                for (int hl = 0; hl < G; hl++) d[hl] = 0.f;
                for (int i = sgs[gr]; i < sgs[gr + 1]; i++) {
                    const float cf = (float)((krows[(i - 1) * R + boff] >> sh) & CMASK);
#pragma unroll
                    for (int hl = 0; hl < G; hl++) d[hl] = fmaf(sq[i * G + hl], cf, d[hl]);
                }
                const uint32_t sz = kmeta[meta_word(gr, t)];
                const float sg = h2f_lo(sz), zg = h2f_hi(sz);
#pragma unroll
                for (int hl = 0; hl < G; hl++) sc[hl] = fmaf(sg, d[hl], fmaf(zg, sqg[gr * G + hl], sc[hl]));
            }
#pragma unroll
            for (int hl = 0; hl < G; hl++) {
                sc[hl] = valid ? sc[hl] * kScoreScaleLog2 : -INFINITY;
                const float wm = warp_max_f(sc[hl]);
                if (lane == 0) sred[warp * G + hl] = wm;
            }
            __syncthreads();
#pragma unroll
            for (int hl = 0; hl < G; hl++) {
                const float bm = fmaxf(fmaxf(sred[hl], sred[G + hl]), fmaxf(sred[2 * G + hl], sred[3 * G + hl]));
                const float mn = fmaxf(m_run[hl], bm);
                const float mu = (mn == -INFINITY) ? 0.f : mn;   // a page with no valid token
                const float alpha = exp2f(m_run[hl] - mu);       // 0 on the first page
                m_run[hl] = mn;
                o_acc[hl] *= alpha;
                l_run[hl] *= alpha;
                sp[t * G + hl] = exp2f(sc[hl] - mu);
            }
            __syncthreads();
        }

        // ---- values: thread c = value channel c
        {
            const int c = tid, vg = c / GS;
            const uint8_t *vrow = vcodes + c * R;
#pragma unroll 1
            for (int tb = 0; tb < R; tb += 4) {
                const uint32_t w = *reinterpret_cast<const uint32_t *>(vrow + tb);
#pragma unroll
                for (int e = 0; e < 32 / BITS; e++) {
                    const int t = tb * PER + e;
                    const uint32_t sz = vmeta[meta_word(vg, t)];
                    const float v = fmaf(h2f_lo(sz), (float)((w >> (e * BITS)) & CMASK), h2f_hi(sz));
#pragma unroll
                    for (int hl = 0; hl < G; hl++) {
                        const float p = sp[t * G + hl];
                        o_acc[hl] = fmaf(p, v, o_acc[hl]);
                        l_run[hl] += p;
                    }
                }
            }
        }
        __syncthreads();
    }
    seg0 = seg1;
    }

    // partial result of this split (an empty split reports m = -inf, l = 0)
#pragma unroll
    for (int hl = 0; hl < G; hl++) {
        const size_t row = ((size_t)b * Hq + (size_t)h * G + hl) * S + s;
        part_o[row * kD + tid] = o_acc[hl];
        if (tid == 0) part_ml[row] = make_float2(m_run[hl], l_run[hl]);
    }
    merge_unit_if_last<G, 128>(part_o, part_ml, S, (size_t)b * Hq + (size_t)h * G, out, counters + unit,
                               reinterpret_cast<float *>(smem), v_rot ? v_rot + (size_t)h * kD * kD : nullptr);
}

template <int BITS, int G, int NG>
cudaError_t launch_simt_t(const kvq_cache &c, int Hq, const int32_t *idx, const float *qsel,
                          const float *qgsum, int k, float *part_o, float2 *part_ml, int S, float *out,
                          cudaStream_t st) {
    const int stage_bytes = (k - 1) * row_bytes(BITS) + fixed_bytes(BITS, NG);
    // the stage area doubles as the scratch of the protected-tier splits and
    // of the split merge
    constexpr int kTierBytes = (tier_scratch_floats(G) * 4 + 15) / 16 * 16;
    constexpr int kMergeBytes = (merge_scratch_floats(G, 128, 256) * 4 + 15) / 16 * 16;
    int stage_area = max(2 * stage_bytes, kMergeBytes);
    if (tier_ctas(c)) stage_area = max(stage_area, kTierBytes);
    const size_t smem = (size_t)stage_area + SimtSmem<G>::extra;
    constexpr int kMaxStages = 2 * (127 * row_bytes(BITS) + fixed_bytes(BITS, NG));
    constexpr int kMaxArea = kMaxStages > kTierBytes ? (kMaxStages > kMergeBytes ? kMaxStages : kMergeBytes)
                                                     : (kTierBytes > kMergeBytes ? kTierBytes : kMergeBytes);
    constexpr int kMaxSmem = kMaxArea + SimtSmem<G>::extra;
    static std::atomic<uint64_t> done{0};
    auto fn = decode_simt_kernel<BITS, G, NG>;
    cudaError_t e = set_smem_once(fn, kMaxSmem, done);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)S, (unsigned)c.n_kv_heads, (unsigned)c.batch);
    fn<<<grid, 128, smem, st>>>(static_cast<const uint8_t *>(c.pages), c.seq_len, c.n_kv_heads,
                                c.capacity / kT, Hq, idx, qsel, qgsum, k, part_o, part_ml, S, out,
                                unit_counter(c, 0, 0), c.status, c.n_sink, c.n_recent, stage_area, c.v_rot,
                                buckets_of(c), c.bucket / kT);
    return cudaGetLastError();
}

}  // namespace

// merge of the split partials: out = sum_s e^{m_s-M} o_s / sum_s e^{m_s-M} l_s
__global__ void __launch_bounds__(128)
combine_kernel(const float *__restrict__ part_o, const float2 *__restrict__ part_ml, int S,
               float *__restrict__ out) {
    const size_t row = blockIdx.x;            // (b, h) flattened
    const int c = threadIdx.x;
    const float2 *ml = part_ml + row * S;
    float M = -INFINITY;
    for (int s = 0; s < S; s++) M = fmaxf(M, ml[s].x);
    float acc = 0.f, L = 0.f;
    if (M != -INFINITY) {
        for (int s = 0; s < S; s++) {
            const float2 v = ml[s];
            const float w = exp2f(v.x - M);   // empty splits: exp2(-inf) = 0
            L = fmaf(w, v.y, L);
            acc = fmaf(w, part_o[(row * S + s) * kD + c], acc);
        }
    }
    out[row * kD + c] = (L > 0.f) ? acc / L : 0.f;
}

cudaError_t launch_decode_simt(const kvq_cache &c, int Hq, const int32_t *idx, const float *qsel,
                               const float *qgsum, int k, float *part_o, float2 *part_ml, int S,
                               float *out, cudaStream_t st) {
    const int g = Hq / c.n_kv_heads;
    const int ng = groups_of(c);
#define KVQ_SIMT_CASE(BITS, G)                                                                          \
    if (c.bits == BITS && g == G)                                                                       \
        return ng == 1 ? launch_simt_t<BITS, G, 1>(c, Hq, idx, qsel, qgsum, k, part_o, part_ml, S, out, st) \
                       : launch_simt_t<BITS, G, kNG>(c, Hq, idx, qsel, qgsum, k, part_o, part_ml, S, out, st);
    KVQ_SIMT_CASE(2, 1) KVQ_SIMT_CASE(2, 2) KVQ_SIMT_CASE(2, 4) KVQ_SIMT_CASE(2, 8)
    KVQ_SIMT_CASE(4, 1) KVQ_SIMT_CASE(4, 2) KVQ_SIMT_CASE(4, 4) KVQ_SIMT_CASE(4, 8)
#undef KVQ_SIMT_CASE
    return cudaErrorInvalidValue;
}

cudaError_t launch_combine(int rows, const float *part_o, const float2 *part_ml, int S, float *out,
                           cudaStream_t st) {
    combine_kernel<<<(unsigned)rows, 128, 0, st>>>(part_o, part_ml, S, out);
    return cudaGetLastError();
}

}  // namespace kvq
