// kvq_append: key transform, channel-0 protection, group min/max quantization
// and channel-major packing into 128-token pages.
//
// "Dual-QK: Sharp Queries and Flat Keys for Prunable 2-bit KV Caches":
//   §3.1 keys are multiplied by the fixed key transform (K' = K A);
//   §3.3 key channel 0 is kept in BF16 and excluded from the quantization
//        range; the remaining channels (and the values) use an asymmetric
//        min/max grid per token; within each 128-token page the codes are
//        stored channel-major, one channel of one page per 32-byte row.
//
// With bucket-relative RoPE (§3.4) each key is first moved into the frame of
// its bucket's anchor (channel pairs (i, i + 64) rotated back by the anchor's
// angle, from the caller's rotary table), then transformed.
//
// With a value rotation (§3.3, App. B.2: values are rotated before they are
// quantized, with the grid clipped to [clip*min, clip*max]; keys are not
// clipped) the values go through the same fixed-order transform as the keys,
// with the rotation in place of A; the protected BF16 copies hold the rotated
// values too.
//
// One CTA = one (sequence, KV head) and a tile of kTile destination positions
// aligned to kTile, so the code bytes a CTA writes belong to it alone; thread
// j owns channel j and warp w owns quantization group w.  The arithmetic is
// float64 with a fixed order (fma chain over the input channel), which makes
// the stored bytes reproducible bit for bit.
#include "kvq_internal.cuh"

#include <cooperative_groups.h>

namespace kvq {
namespace {

constexpr int kTile = 16;   // destination positions per CTA (multiple of 8)

// Merge the kTile codes of one channel row into its packed bytes.
// `valid` has bit tt set for tile positions this call writes.
template <int BITS>
__device__ __forceinline__ void store_row(uint8_t *row_tile, const uint32_t (&codes)[kTile],
                                          uint32_t valid) {
    if constexpr (BITS == 2) {
        uint32_t word = 0, mask = 0;
#pragma unroll
        for (int tt = 0; tt < kTile; tt++) {
            word |= codes[tt] << (2 * tt);
            if (valid >> tt & 1u) mask |= 3u << (2 * tt);
        }
        uint32_t *p = reinterpret_cast<uint32_t *>(row_tile);
        *p = (*p & ~mask) | (word & mask);
    } else {
        unsigned long long word = 0, mask = 0;
#pragma unroll
        for (int tt = 0; tt < kTile; tt++) {
            word |= (unsigned long long)codes[tt] << (4 * tt);
            if (valid >> tt & 1u) mask |= 15ull << (4 * tt);
        }
        unsigned long long *p = reinterpret_cast<unsigned long long *>(row_tile);
        *p = (*p & ~mask) | (word & mask);
    }
}

template <typename Tin, int BITS, int NG>
__global__ void __launch_bounds__(128)
append_kernel(uint8_t *__restrict__ pages, const int32_t *__restrict__ seq_len,
              uint32_t *__restrict__ status, const Tin *__restrict__ K,
              const Tin *__restrict__ V, const double *__restrict__ A, const double *__restrict__ Rv,
              double vclip, int Hkv, int NB, int n_new, int capacity, int n_sink, int n_recent,
              const double *__restrict__ rope, int w) {
    constexpr int R = row_bytes(BITS);
    __shared__ double ks[kTile][kD];
    __shared__ double vs[kTile][kD];
    __shared__ double red[8];                 // block range of one grid per token (NG == 1)

    const int b = blockIdx.z, h = blockIdx.y;
    const int len = seq_len[b];
    if (len < 0 || len + n_new > capacity) {
        if (threadIdx.x == 0) atomicOr(status, (uint32_t)KVQ_DEV_CAPACITY);
        return;
    }
    const int first = (len / kTile) * kTile + blockIdx.x * kTile;
    const int lo = max(first, len), hi = min(first + kTile, len + n_new);
    if (lo >= hi) return;

    // stage the inputs of the tile as float64 (zeros outside [lo, hi))
    const size_t in_base = ((size_t)b * Hkv + h) * (size_t)n_new;
    for (int e = threadIdx.x; e < kTile * kD; e += blockDim.x) {
        const int tt = e / kD, c = e % kD, pos = first + tt;
        double kv = 0.0, vv = 0.0;
        if (pos >= lo && pos < hi) {
            const size_t src = (in_base + (size_t)(pos - len)) * kD + c;
            kv = in_to_double(K[src]);
            vv = in_to_double(V[src]);
        }
        ks[tt][c] = kv;
        vs[tt][c] = vv;
    }
    __syncthreads();
    if (rope) {
        // k T_b for the bucket of each position (thread j < 64: pair (j, j + 64))
        if (threadIdx.x < kD / 2) {
            const double2 *cs = reinterpret_cast<const double2 *>(rope);
#pragma unroll 4
            for (int tt = 0; tt < kTile; tt++) {
                const int pos = first + tt;
                if (pos < lo || pos >= hi) continue;
                rope_unanchor_pair(ks[tt][threadIdx.x], ks[tt][threadIdx.x + kD / 2],
                                   __ldg(cs + (size_t)(pos / w) * (kD / 2) + threadIdx.x));
            }
        }
        __syncthreads();
    }

    const int j = threadIdx.x;          // channel
    const int lane = j & 31;
    const int grp = j >> 5;             // quantization group (= warp)

    // Y[t][j] = sum_c X[t][c] M[c][j], fma chain c = 0..127 from 0.0.  A full
    // tile interleaves its kTile chains (M read once per c); a partial tile (a
    // decode step appends one token) runs only the chains of its tokens.
    auto transform = [&](const double (*xs)[kD], const double *M, double (&acc)[kTile]) {
#pragma unroll
        for (int tt = 0; tt < kTile; tt++) acc[tt] = 0.0;
        const double *Mh = M + (size_t)h * kD * kD + j;
        if (hi - lo == kTile) {
#pragma unroll 4
            for (int c = 0; c < kD; c++) {
                const double a = __ldg(Mh + (size_t)c * kD);
#pragma unroll
                for (int tt = 0; tt < kTile; tt++) acc[tt] = fma(xs[tt][c], a, acc[tt]);
            }
        } else {
#pragma unroll
            for (int tt = 0; tt < kTile; tt++) {
                if (first + tt < lo || first + tt >= hi) continue;     // uniform over the CTA
                double a_reg[8];
                double x = 0.0;
                for (int c0 = 0; c0 < kD; c0 += 8) {
#pragma unroll
                    for (int u = 0; u < 8; u++) a_reg[u] = __ldg(Mh + (size_t)(c0 + u) * kD);
#pragma unroll
                    for (int u = 0; u < 8; u++) x = fma(xs[tt][c0 + u], a_reg[u], x);
                }
                acc[tt] = x;
            }
        }
    };
    double acc[kTile];
    transform(ks, A, acc);                  // K' = K A
    if (Rv) {
        // V Rv, written back over the tile's values once every chain has read them
        double vacc[kTile];
        transform(vs, Rv, vacc);
        __syncthreads();
#pragma unroll
        for (int tt = 0; tt < kTile; tt++) vs[tt][j] = vacc[tt];
    }

    uint8_t *page = pages + (((size_t)b * Hkv + h) * NB + (size_t)(first / kT)) * page_bytes(BITS, NG);
    const int t0 = first % kT;
    uint32_t valid = 0;
#pragma unroll
    for (int tt = 0; tt < kTile; tt++)
        if (first + tt >= lo && first + tt < hi) valid |= 1u << tt;

    uint16_t *ch0 = reinterpret_cast<uint16_t *>(page + off_ch0(BITS));
    uint32_t *kmeta = reinterpret_cast<uint32_t *>(page + off_kmeta(BITS));
    uint32_t *vmeta = reinterpret_cast<uint32_t *>(page + off_vmeta(BITS, NG));
    // groups of 32 (NG = 4): warp = group; one grid per token (NG = 1): the CTA
    const int mg = NG == 1 ? 0 : grp;                   // metadata group of this thread
    const bool writes_meta = NG == 1 ? j == 0 : lane == 0;
    auto quantize = [&](double x, bool in_range, uint16_t &sb, uint16_t &zb) -> uint32_t {
        if constexpr (NG == 1) return quantize_block128<BITS>(x, in_range, red, sb, zb);
        else return quantize_lane<BITS>(x, in_range, sb, zb);
    };
    auto quantize_v = [&](double x, uint16_t &sb, uint16_t &zb) -> uint32_t {
        if constexpr (NG == 1) return quantize_block128<BITS>(x, true, red, sb, zb, vclip);
        else return quantize_lane<BITS>(x, true, sb, zb, vclip);
    };

    // keys: channel 0 -> bf16; group 0 starts at channel 1
    uint32_t codes[kTile];
#pragma unroll
    for (int tt = 0; tt < kTile; tt++) {
        uint16_t sb, zb;
        codes[tt] = 0;
        if (!(valid >> tt & 1u)) continue;                        // uniform over the CTA
        codes[tt] = quantize(acc[tt], j != 0, sb, zb);
        if (writes_meta) kmeta[meta_word(mg, t0 + tt)] = (uint32_t)sb | ((uint32_t)zb << 16);
        if (j == 0) ch0[t0 + tt] = __bfloat16_as_ushort(__double2bfloat16(acc[tt]));
    }
    if (j != 0) store_row<BITS>(page + (size_t)j * R + t0 * BITS / 8, codes, valid);

    // values (rotated when Rv is given; thread j reads only its own channel
    // from here on), grids clipped by vclip
#pragma unroll
    for (int tt = 0; tt < kTile; tt++) {
        uint16_t sb, zb;
        codes[tt] = 0;
        if (!(valid >> tt & 1u)) continue;
        codes[tt] = quantize_v(vs[tt][j], sb, zb);
        if (writes_meta) vmeta[meta_word(mg, t0 + tt)] = (uint32_t)sb | ((uint32_t)zb << 16);
    }
    store_row<BITS>(page + off_vcodes(BITS) + (size_t)j * R + t0 * BITS / 8, codes, valid);

    // protected tier: BF16 copies of sink tokens and of the last n_recent
    // tokens of the sequence once this append completes
    if (n_sink + n_recent > 0) {
        uint16_t *slots = reinterpret_cast<uint16_t *>(
            unit_slots(pages, gridDim.z, Hkv, NB, BITS, (size_t)b * Hkv + h, n_sink + n_recent, NG));
#pragma unroll
        for (int tt = 0; tt < kTile; tt++) {
            const int pos = first + tt;
            if (!(valid >> tt & 1u) || !stores_slot(pos, len + n_new, n_sink, n_recent)) continue;
            uint16_t *dst = slots + (size_t)slot_of(pos, n_sink, n_recent) * (kSlotBytes / 2);
            dst[j] = __bfloat16_as_ushort(__double2bfloat16(acc[tt]));
            dst[kD + j] = __bfloat16_as_ushort(__double2bfloat16(vs[tt][j]));
        }
    }
}

// Appends of a few tokens (a decode step adds one): one CTA per (sequence,
// KV head, quantization group), so the key transform's columns -- and the
// reads of A they need, 32 KB per CTA, staged with one cp.async burst -- are
// spread over 4 * n_kv_heads * batch SMs.  Warp w transforms and quantizes new
// token w (lane = channel of the group); the codes then go through shared
// memory to one thread per channel row, which merges the new tokens into the
// packed bytes in order (neighbouring tokens share bytes).  With a value
// rotation the same staging memory then takes the group's 32 columns of the
// rotation for the values' chains.  The four CTAs of a (sequence, KV head)
// form a cluster: with one grid per token (NG = 1) each token's key and value
// ranges are met over the four CTAs' warps through distributed shared memory.
// The last CTA of a sequence to finish advances its length, using the
// sequence's completion counter in the status array.
constexpr int kSmallMax = 4;

template <typename Tin, int BITS, int NG>
__global__ void __cluster_dims__(kNG, 1, 1) __launch_bounds__(128)
append_small_kernel(uint8_t *__restrict__ pages, int32_t *__restrict__ seq_len,
                    uint32_t *__restrict__ status, const Tin *__restrict__ K,
                    const Tin *__restrict__ V, const double *__restrict__ A, const double *__restrict__ Rv,
                    double vclip, int Hkv, int NB, int n_new, int capacity, int n_sink, int n_recent,
                    const double *__restrict__ rope, int w_tok, int advance) {
    constexpr int R = row_bytes(BITS);
    constexpr int PER = 8 / BITS;
    // a decode step's channel choice may start meanwhile (it reads nothing
    // this kernel writes, and waits for it before it exits)
    asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
    static_assert(kSmallMax * 32 == 128, "one warp per new token");
    __shared__ __align__(16) double As[kD][kGroup];        // A[:, 32 grp .. 32 grp + 31], then Rv[...]
    __shared__ double ks[kSmallMax][kD];
    __shared__ double vsd[kSmallMax][kD];                  // full value rows (value rotation only)
    __shared__ uint8_t kcode[kSmallMax][kGroup];
    __shared__ uint8_t vcode[kSmallMax][kGroup];
    __shared__ double trange[kSmallMax][4];                // NG = 1: this CTA's {key lo, hi, value lo, hi}
    __shared__ int s_len;
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();

    const int grp = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int t = threadIdx.x, lane = t & 31, w = t >> 5;
    const int j = grp * kGroup + lane;                     // this lane's channel
    const double *Ah = A + (size_t)h * kD * kD + grp * kGroup;
    for (int e = t; e < kD * kGroup / 2; e += 128) {
        const int c = e >> 4, part = e & 15;
        cp_async16(&As[c][2 * part], Ah + (size_t)c * kD + 2 * part);
    }
    cp_async_commit();
    const size_t in_base = ((size_t)b * Hkv + h) * (size_t)n_new;
    for (int e = t; e < n_new * kD; e += 128) ks[e / kD][e % kD] = in_to_double(K[in_base * kD + e]);
    if (Rv)
        for (int e = t; e < n_new * kD; e += 128) vsd[e / kD][e % kD] = in_to_double(V[in_base * kD + e]);
    double v = (w < n_new) ? in_to_double(V[(in_base + w) * kD + j]) : 0.0;
    if (t == 0) s_len = seq_len[b];
    cp_async_wait<0>();
    __syncthreads();
    const int len = s_len;
    const bool ok = len >= 0 && len + n_new <= capacity;
    uint8_t *unit = pages + ((size_t)b * Hkv + h) * NB * (size_t)page_bytes(BITS, NG);
    if (rope && ok) {
        // k T_b for the bucket of each new position
        const double2 *cs = reinterpret_cast<const double2 *>(rope);
        for (int e = t; e < n_new * (kD / 2); e += 128) {
            const int i = e / (kD / 2), c = e % (kD / 2);
            rope_unanchor_pair(ks[i][c], ks[i][c + kD / 2], __ldg(cs + (size_t)((len + i) / w_tok) * (kD / 2) + c));
        }
        __syncthreads();
    }

    // K'[t][j] = sum_c K[t][c] A[c][j], fma chain c = 0..127 from 0.0
    double x = 0.0;
    if (ok && w < n_new) {
#pragma unroll 16
        for (int c = 0; c < kD; c++) x = fma(ks[w][c], As[c][lane], x);
    }
    if (Rv) {
        // the same chain for the rotated value, (V Rv)[t][j], with the
        // group's columns of Rv staged over those of A
        __syncthreads();
        const double *Rh = Rv + (size_t)h * kD * kD + grp * kGroup;
        for (int e = t; e < kD * kGroup / 2; e += 128) {
            const int c = e >> 4, part = e & 15;
            cp_async16(&As[c][2 * part], Rh + (size_t)c * kD + 2 * part);
        }
        cp_async_commit();
        cp_async_wait<0>();
        __syncthreads();
        if (ok && w < n_new) {
            double y = 0.0;
#pragma unroll 16
            for (int c = 0; c < kD; c++) y = fma(vsd[w][c], As[c][lane], y);
            v = y;
        }
    }

    // one grid per token: the token's ranges over all four CTAs of the cluster
    double klo = 0.0, khi = 0.0, vlo = 0.0, vhi = 0.0;
    if constexpr (NG == 1) {
        if (ok && w < n_new) {
            const double a = warp_min(j != 0 ? x : pos_inf()), bk = warp_max(j != 0 ? x : neg_inf());
            const double c = warp_min(v), d = warp_max(v);
            if (lane == 0) {
                trange[w][0] = a;
                trange[w][1] = bk;
                trange[w][2] = c;
                trange[w][3] = d;
            }
        }
        cluster.sync();
        if (ok && w < n_new) {
            klo = pos_inf(), khi = neg_inf(), vlo = pos_inf(), vhi = neg_inf();
#pragma unroll
            for (int rr = 0; rr < kNG; rr++) {
                const double *pr = cluster.map_shared_rank(&trange[w][0], rr);
                klo = fmin(klo, pr[0]);
                khi = fmax(khi, pr[1]);
                vlo = fmin(vlo, pr[2]);
                vhi = fmax(vhi, pr[3]);
            }
        }
        cluster.sync();                                    // the peers are done reading trange
    }

    if (ok && w < n_new) {                                 // uniform over the warp
        const int pos = len + w, tt = pos % kT;
        uint8_t *page = unit + (size_t)(pos / kT) * page_bytes(BITS, NG);
        const int mg = NG == 1 ? 0 : grp;                  // metadata group
        const bool meta_writer = lane == 0 && (NG != 1 || grp == 0);
        uint16_t sb, zb;
        kcode[w][lane] = (uint8_t)(NG == 1 ? code_in_range<BITS>(x, klo, khi, sb, zb)
                                           : quantize_lane<BITS>(x, j != 0, sb, zb));
        if (meta_writer)
            reinterpret_cast<uint32_t *>(page + off_kmeta(BITS))[meta_word(mg, tt)] = (uint32_t)sb | ((uint32_t)zb << 16);
        if (j == 0) reinterpret_cast<uint16_t *>(page + off_ch0(BITS))[tt] = __bfloat16_as_ushort(__double2bfloat16(x));
        vcode[w][lane] = (uint8_t)(NG == 1 ? code_in_range<BITS>(v, __dmul_rn(vclip, vlo), __dmul_rn(vclip, vhi), sb, zb)
                                           : quantize_lane<BITS>(v, true, sb, zb, vclip));
        if (meta_writer)
            reinterpret_cast<uint32_t *>(page + off_vmeta(BITS, NG))[meta_word(mg, tt)] = (uint32_t)sb | ((uint32_t)zb << 16);
        // protected tier: BF16 copies (sink tokens, the last n_recent tokens)
        if (n_sink + n_recent > 0 && stores_slot(pos, len + n_new, n_sink, n_recent)) {
            uint16_t *dst = reinterpret_cast<uint16_t *>(
                unit_slots(pages, gridDim.z, Hkv, NB, BITS, (size_t)b * Hkv + h, n_sink + n_recent, NG) +
                (size_t)slot_of(pos, n_sink, n_recent) * kSlotBytes);
            dst[j] = __bfloat16_as_ushort(__double2bfloat16(x));
            dst[kD + j] = __bfloat16_as_ushort(__double2bfloat16(v));
        }
    }
    __syncthreads();
    if (ok && t < 2 * kGroup) {
        // thread t < 32: key row of channel j; 32 <= t < 64: value row
        const bool val = t >= kGroup;
        if (val || j != 0) {
            for (int i = 0; i < n_new; i++) {
                const int pos = len + i, tt = pos % kT;
                const int byte = tt / PER, sh = (tt % PER) * BITS;
                uint8_t *p = unit + (size_t)(pos / kT) * page_bytes(BITS, NG) + (val ? off_vcodes(BITS) : 0) +
                             (size_t)j * R + byte;
                const uint8_t clear = (uint8_t)~(((1u << BITS) - 1u) << sh);
                const uint32_t code = val ? vcode[i][lane] : kcode[i][lane];
                *p = (uint8_t)((*p & clear) | (code << sh));
            }
        }
    } else if (!ok && t == 0) {
        atomicOr(status, (uint32_t)KVQ_DEV_CAPACITY);
    }

    __syncthreads();
    if (advance && t == 0) {
        __threadfence();
        const unsigned prev = atomicAdd(status + 1 + b, 1u);
        if (prev == (unsigned)(Hkv * kNG) - 1u) {   // every CTA of sequence b has read its length
            if (ok) seq_len[b] = len + n_new;
            atomicExch(status + 1 + b, 0u);
        }
    }
}

__global__ void advance_kernel(int32_t *seq_len, int B, int n_new, int capacity) {
    const int b = blockIdx.x * blockDim.x + threadIdx.x;
    if (b < B) {
        const int len = seq_len[b];
        if (len >= 0 && len + n_new <= capacity) seq_len[b] = len + n_new;
    }
}

template <typename Tin, int BITS, int NG>
cudaError_t launch_append_t(const kvq_cache &c, const void *K, const void *V, int n_new,
                            const double *A, cudaStream_t st, bool advance = true) {
    const double *Rv = c.v_rot;
    const double vclip = value_clip(c);
    const double *rope = c.bucket > 0 ? c.rope : nullptr;
    const int NB = c.capacity / kT;
    // a few tokens: one CTA per 32-channel group (a cluster of four per
    // sequence and KV head); a prefill: the tile kernel and the length advance
    if (n_new <= kSmallMax) {
        dim3 grid((unsigned)kNG, (unsigned)c.n_kv_heads, (unsigned)c.batch);
        append_small_kernel<Tin, BITS, NG><<<grid, 128, 0, st>>>(
            static_cast<uint8_t *>(c.pages), c.seq_len, c.status, static_cast<const Tin *>(K),
            static_cast<const Tin *>(V), A, Rv, vclip, c.n_kv_heads, NB, n_new, c.capacity, c.n_sink, c.n_recent,
            rope, c.bucket, advance ? 1 : 0);
        return cudaGetLastError();
    }
    dim3 grid((unsigned)((n_new + kTile - 1) / kTile + 1), (unsigned)c.n_kv_heads, (unsigned)c.batch);
    append_kernel<Tin, BITS, NG><<<grid, 128, 0, st>>>(
        static_cast<uint8_t *>(c.pages), c.seq_len, c.status, static_cast<const Tin *>(K),
        static_cast<const Tin *>(V), A, Rv, vclip, c.n_kv_heads, NB, n_new, c.capacity, c.n_sink, c.n_recent,
        rope, c.bucket);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    advance_kernel<<<(c.batch + 127) / 128, 128, 0, st>>>(c.seq_len, c.batch, n_new, c.capacity);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_append_adv(const kvq_cache &c, const void *K, const void *V, int dtype, int n_new,
                              const double *A, cudaStream_t st, bool advance) {
    const bool one = groups_of(c) == 1;
#define KVQ_APPEND_CASE(TIN, BITS)                                                              \
    if (c.bits == BITS)                                                                        \
        return one ? launch_append_t<TIN, BITS, 1>(c, K, V, n_new, A, st, advance)             \
                   : launch_append_t<TIN, BITS, kNG>(c, K, V, n_new, A, st, advance);
    if (dtype == KVQ_DTYPE_F32) {
        KVQ_APPEND_CASE(float, 2)
        KVQ_APPEND_CASE(float, 4)
    } else {
        KVQ_APPEND_CASE(uint16_t, 2)
        KVQ_APPEND_CASE(uint16_t, 4)
    }
#undef KVQ_APPEND_CASE
    return cudaErrorInvalidValue;
}

cudaError_t launch_append(const kvq_cache &c, const void *K, const void *V, int dtype, int n_new,
                          const double *A, cudaStream_t st) {
    return launch_append_adv(c, K, V, dtype, n_new, A, st, true);
}

// The append of a decode step whose length the step's decode advances: at
// most kSmallMax tokens, the small-append kernel without its length advance;
// the step's channel choice is launched after it as its programmatic
// dependent.
cudaError_t launch_step_append(const kvq_cache &c, const void *K, const void *V, int dtype, int n_new,
                               const double *A, cudaStream_t st) {
    if (n_new < 1 || n_new > kSmallMax) return cudaErrorInvalidValue;
    return launch_append_adv(c, K, V, dtype, n_new, A, st, false);
}

}  // namespace kvq
