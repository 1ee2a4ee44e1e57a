// Internal definitions shared by the kvq CUDA kernels (sm_100a).
// Page layout and arithmetic conventions are documented in include/kvq.h.
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <atomic>

#include "kvq.h"

namespace kvq {

constexpr int kD = 128;        // head dimension
constexpr int kT = 128;        // tokens per page
constexpr int kGroup = 32;     // channels per quantization group
constexpr int kNG = kD / kGroup;

// Page layout for `bits`-wide codes and `ng` quantization groups per head
// (4: groups of 32 channels; 1: the pages' one grid per token).
__host__ __device__ constexpr int row_bytes(int bits) { return kT * bits / 8; }
__host__ __device__ constexpr int off_vcodes(int bits) { return 128 * row_bytes(bits); }
__host__ __device__ constexpr int off_ch0(int bits) { return 256 * row_bytes(bits); }
__host__ __device__ constexpr int meta_bytes(int ng) { return 4 * kT * ng; }
__host__ __device__ constexpr int off_kmeta(int bits) { return off_ch0(bits) + 256; }
__host__ __device__ constexpr int off_vmeta(int bits, int ng = kNG) { return off_kmeta(bits) + meta_bytes(ng); }
__host__ __device__ constexpr int page_bytes(int bits, int ng = kNG) { return off_vmeta(bits, ng) + meta_bytes(ng); }
// word index of the {scale, zero} pair of token t (0..127), group g (0..3)
// inside a page's key or value metadata block (chunks of 4 tokens are stored
// XOR-permuted within blocks of 8 chunks, see include/kvq.h)
__host__ __device__ constexpr int meta_word(int g, int t) {
    return 128 * g + 4 * ((t >> 2) ^ (((t >> 5) & 3) ^ ((g & 1) << 2))) + (t & 3);
}
// bytes from the value codes to the end of the page: what every decode step
// reads in full (value codes, channel 0, key and value metadata)
__host__ __device__ constexpr int fixed_bytes(int bits, int ng = kNG) { return page_bytes(bits, ng) - off_vcodes(bits); }
// groups per head of a cache (group = 32 or 128 channels)
inline int groups_of(const kvq_cache &c) { return kD / c.group; }
// clipping ratio of the value grids (0 in the descriptor: none)
inline double value_clip(const kvq_cache &c) { return c.v_clip == 0.0 ? 1.0 : c.v_clip; }
// RoPE buckets of a cache (1 without buckets): entries of every selection array
inline int buckets_of(const kvq_cache &c) { return c.bucket > 0 ? (c.capacity + c.bucket - 1) / c.bucket : 1; }

// Bucket-relative RoPE (Dual-QK §3.4): move channel pair (x_i, x_{i+64}) of a
// post-RoPE vector into the frame of a bucket anchor, i.e. rotate it by
// -a*theta_i given cs = {cos, sin} of a*theta_i; each product rounded, then
// the sum or difference (no contraction), the definition both the library
// and its tests use.
__device__ __forceinline__ void rope_unanchor_pair(double &xi, double &xj, double2 cs) {
    const double a = xi, b = xj;
    xi = __dadd_rn(__dmul_rn(a, cs.x), __dmul_rn(b, cs.y));
    xj = __dsub_rn(__dmul_rn(b, cs.x), __dmul_rn(a, cs.y));
}

// ------------------------------------------------------------ protected tier
// slot of the protected BF16 tier: 128 bf16 of K' then 128 bf16 of V
constexpr int kSlotBytes = 2 * kD * 2;
// protected set of a sequence of length len: [0, sink_end) and [recent_start, len);
// the codes are read for [sink_end, recent_start)
struct Tier {
    int sink_end, recent_start;
};
__host__ __device__ inline Tier tier_of(int len, int n_sink, int n_recent) {
    const int se = len < n_sink ? len : n_sink;
    int rs = len - n_recent;
    if (rs < se) rs = se;
    return {se, rs};
}
__host__ __device__ inline int slot_of(int pos, int n_sink, int n_recent) {
    return pos < n_sink ? pos : n_sink + pos % n_recent;
}
// a new token gets its slot when it is a sink token or among the last n_recent
// of the sequence once the append completes (length len_after)
__host__ __device__ inline bool stores_slot(int pos, int len_after, int n_sink, int n_recent) {
    return pos < n_sink || (n_recent > 0 && pos >= len_after - n_recent);
}
// the unit's slots: after every page of the cache
__host__ __device__ inline uint8_t *unit_slots(void *pages, int B, int Hkv, int NB, int bits, size_t unit, int NP,
                                               int ng = kNG) {
    return static_cast<uint8_t *>(pages) + (size_t)B * Hkv * NB * page_bytes(bits, ng) + unit * (size_t)NP * kSlotBytes;
}
// extra CTAs per (sequence, KV head) of a decode that handle the tier
inline int tier_ctas(const kvq_cache &c) { return c.n_sink + c.n_recent > 0 ? 2 : 0; }

// log2(e) / sqrt(128): scores are kept in the base-2 exponent domain
constexpr float kScoreScaleLog2 = 0.12751743074460787f;

// ------------------------------------------------------------ channel choice
// How many of channels i0 .. i0 + N - 1 (channel 0 left out) come before
// channel j in the order (energy descending, index ascending).  `key` holds
// the 128 energies' bit patterns: energies are >= 0, so the patterns order
// like the values and integer compares decide exactly.  The keys are read
// eight at a time, ahead of their compares.
template <int N>
__device__ __forceinline__ int rank_count(const unsigned long long *key, int j, int i0) {
    static_assert(N % 8 == 0, "keys are read eight at a time");
    const unsigned long long kj = key[j];
    int rk = 0;
#pragma unroll
    for (int b = 0; b < N / 8; b++) {
        unsigned long long v[8];
#pragma unroll
        for (int u = 0; u < 8; u++) v[u] = key[i0 + 8 * b + u];
#pragma unroll
        for (int u = 0; u < 8; u++) {
            const int i = i0 + 8 * b + u;
            rk += (int)((i != 0) & ((v[u] > kj) | ((v[u] == kj) & (i < j))));
        }
    }
    return rk;
}
// the same over channels 64*half .. 64*half + 63
__device__ __forceinline__ int rank_half(const unsigned long long *key, int j, int half) {
    return rank_count<64>(key, j, 64 * half);
}

// ------------------------------------------------------------ page plan
// What the tensor-core decode (INT2, four query heads per KV head) needs of
// one channel choice, in the order its shared memory holds it.  A decode
// step's preparation kernel writes one per (sequence, KV head, RoPE bucket)
// into the workspace; the decode copies it in after waiting for that kernel.
// The three-call decode builds the same plan from the channel list.
constexpr int kPlanChunks = 64;                   // 64-byte chunks of a page's key rows
constexpr int kPlanCopies = kPlanChunks / 2 + 2;  // runs after gap filling, plus the tail
struct __align__(16) PagePlan {
    uint2 bq[8][32];          // score-MMA B fragments per k-step and lane
    float q0[4];              // channel 0's q' per head (fp32, as in qsel)
    float qg[4][kNG];         // zero-point sums per head and key group (as in qgsum)
    uint2 copy[kPlanCopies];  // {byte offset in the page, bytes}; the last one is the page tail
    uint32_t tx_keys;         // bytes of the key-chunk copies of one page
    int n_copies;
    uint32_t pad[2];
};
static_assert(sizeof(PagePlan) % 16 == 0, "plans are copied in 16-byte pieces");

// fp16 hi/lo split of a float: hi = fp16(x), lo = fp16(x - hi)
__device__ __forceinline__ uint16_t f16_part(float x, int part) {
    const __half hi = __float2half_rn(x);
    if (part == 0) return __half_as_ushort(hi);
    return __half_as_ushort(__float2half_rn(x - __half2float(hi)));
}
// B fragment word of k-step ks, lane, register half rr of the score MMAs:
// column gid = lane / 4 is (head gid / 2, fp16 part gid % 2); k-slots 2tig,
// 2tig+1 (rr = 0) and 2tig+8, 2tig+9 (rr = 1) are channels 16ks + tig + 8rr
// and that + 4 (this order makes the code loads bank-conflict free).
// `qf(c)` is the fp32 q' of channel c for the column's head, 0 for channel 0
// and for channels that are not selected.
template <typename QF>
__device__ __forceinline__ uint32_t plan_bq_word(int ks, int lane, int rr, QF &&qf) {
    const int gid = lane >> 2, tig = lane & 3, part = gid & 1;
    const int c0 = 16 * ks + tig + 8 * rr, c1 = c0 + 4;
    return (uint32_t)f16_part(qf(gid >> 1, c0), part) | ((uint32_t)f16_part(qf(gid >> 1, c1), part) << 16);
}
// The copy list of a plan from T, the 64-byte chunks of key rows that hold a
// selected row (channel 0's row is never read): runs of chunks in ascending
// order, single unselected chunks between two selected ones filled in (one
// copy instead of two); then the page tail (value codes, channel 0,
// metadata).  Called by a whole warp: lane l looks at chunks 2l and 2l + 1
// as run starts.
__device__ __forceinline__ void plan_copies_warp(PagePlan &p, uint64_t T, int ng, int lane) {
    const uint64_t M = T | ((T << 1) & (T >> 1));
    const uint64_t starts = M & ~(M << 1);
#pragma unroll
    for (int h = 0; h < 2; h++) {
        const int st = 2 * lane + h;
        if ((starts >> st) & 1ull) {
            const int n = __popcll(starts & ((1ull << st) - 1ull));
            const uint64_t inv = ~(M >> st);
            const int len = inv ? __ffsll((long long)inv) - 1 : kPlanChunks - st;
            p.copy[n] = make_uint2(64u * (uint32_t)st, 64u * (uint32_t)len);
        }
    }
    if (lane == 0) {
        const int n = __popcll(starts);
        p.copy[n] = make_uint2((uint32_t)off_vcodes(2), (uint32_t)fixed_bytes(2, ng));
        p.n_copies = n + 1;
        p.tx_keys = 64u * (uint32_t)__popcll(M);
    }
}
// chunk mask from the 128-bit channel choice (word w = channels 32w..32w+31)
__device__ __forceinline__ uint64_t plan_chunks(const uint32_t (&msk)[4]) {
    uint64_t T = 0;
#pragma unroll
    for (int w = 0; w < 4; w++) {
        uint32_t x = w == 0 ? (msk[0] & ~1u) : msk[w];
        x = (x | (x >> 1)) & 0x55555555u;       // chunk bit at each even position
        x = (x | (x >> 1)) & 0x33333333u;       // then compressed to 16 bits
        x = (x | (x >> 2)) & 0x0f0f0f0fu;
        x = (x | (x >> 4)) & 0x00ff00ffu;
        x = (x | (x >> 8)) & 0x0000ffffu;
        T |= (uint64_t)x << (16 * w);
    }
    return T;
}

// ------------------------------------------------------------ conversions
__device__ __forceinline__ double in_to_double(float x) { return (double)x; }
__device__ __forceinline__ double in_to_double(uint16_t bf) {
    return (double)__uint_as_float(((uint32_t)bf) << 16);
}
__device__ __forceinline__ float in_to_float(float x) { return x; }
__device__ __forceinline__ float in_to_float(uint16_t bf) {
    return __uint_as_float(((uint32_t)bf) << 16);
}

// ------------------------------------------------------------ quantization
__device__ __forceinline__ double warp_min(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmin(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ double warp_max(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmax(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// Quantize value x of this lane against the group range (lanes of the warp;
// `in_range` false leaves the lane out of min/max).  Returns the code and,
// through s_bits / z_bits, the fp16 scale / zero-point bit patterns.
// Code of x on the grid of a group with range [lo, hi]: zero = fp16(lo),
// scale = fp16((hi - lo) / (2^BITS - 1)), code = clamp(rint((x - zero) / scale)).
template <int BITS>
__device__ __forceinline__ uint32_t code_in_range(double x, double lo, double hi, uint16_t &s_bits,
                                                  uint16_t &z_bits) {
    constexpr int L = (1 << BITS) - 1;
    const __half zh = __double2half(lo);
    const __half sh = __double2half((hi - lo) / (double)L);
    z_bits = __half_as_ushort(zh);
    s_bits = __half_as_ushort(sh);
    const double z = (double)__half2float(zh);
    const double s = (double)__half2float(sh);
    if (s == 0.0) return 0u;
    double r = rint((x - z) / s);
    r = fmin(fmax(r, 0.0), (double)L);
    return (uint32_t)r;
}
__device__ __forceinline__ double pos_inf() { return __longlong_as_double(0x7ff0000000000000LL); }
__device__ __forceinline__ double neg_inf() { return __longlong_as_double(0xfff0000000000000LL); }

// The grid of a warp's 32 values (lane = channel).  With a clipping ratio
// `clip` (values, Dual-QK App. B.2) the grid spans [clip*min, clip*max]; the
// products are rounded on their own (no contraction into the subtraction),
// and clip = 1 leaves the range as it is.
template <int BITS>
__device__ __forceinline__ uint32_t quantize_lane(double x, bool in_range, uint16_t &s_bits,
                                                  uint16_t &z_bits, double clip = 1.0) {
    const double lo = __dmul_rn(clip, warp_min(in_range ? x : pos_inf()));
    const double hi = __dmul_rn(clip, warp_max(in_range ? x : neg_inf()));
    return code_in_range<BITS>(x, lo, hi, s_bits, z_bits);
}
// The same over all 128 threads of a CTA (thread = channel; one grid per
// token).  Called by every thread; `red` is shared memory of 8 doubles that
// no other code uses between the barriers of two calls.
template <int BITS>
__device__ __forceinline__ uint32_t quantize_block128(double x, bool in_range, double *red, uint16_t &s_bits,
                                                      uint16_t &z_bits, double clip = 1.0) {
    const int w = threadIdx.x >> 5;
    const double lo_w = warp_min(in_range ? x : pos_inf());
    const double hi_w = warp_max(in_range ? x : neg_inf());
    __syncthreads();                                     // the previous call's reads of red are done
    if ((threadIdx.x & 31) == 0) {
        red[w] = lo_w;
        red[4 + w] = hi_w;
    }
    __syncthreads();
    const double lo = __dmul_rn(clip, fmin(fmin(red[0], red[1]), fmin(red[2], red[3])));
    const double hi = __dmul_rn(clip, fmax(fmax(red[4], red[5]), fmax(red[6], red[7])));
    return code_in_range<BITS>(x, lo, hi, s_bits, z_bits);
}

// ------------------------------------------------------------ cp.async
__device__ __forceinline__ void cp_async16(void *smem_dst, const void *gmem_src) {
    uint32_t d = (uint32_t)__cvta_generic_to_shared(smem_dst);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(d), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory"); }
// wait until at most `pending` (0..4) of this thread's commit groups are in flight
__device__ __forceinline__ void cp_async_wait_upto(int pending) {
    if (pending >= 4) cp_async_wait<4>();
    else if (pending == 3) cp_async_wait<3>();
    else if (pending == 2) cp_async_wait<2>();
    else if (pending == 1) cp_async_wait<1>();
    else cp_async_wait<0>();
}

// ------------------------------------------------------------ bulk copies, mbarriers
__device__ __forceinline__ uint32_t smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(bar), "r"(count) : "memory");
}
// expect bytes without arriving (the arrival comes with the key copies)
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;\n" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n"
                 ::"r"(dst), "l"(src), "r"(bytes), "r"(bar) : "memory");
}
// bring `bytes` (a multiple of 16, 16-byte aligned) of global memory into L2
__device__ __forceinline__ void prefetch_l2(const void *src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;\n" ::"l"(src), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
    return ok != 0;
}
__device__ __forceinline__ bool mbar_test_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
    return ok != 0;
}

// Wait for a phase of a barrier with bulk copies on it.  The wait is bounded: after `polls` polls the
// device status word gets KVQ_DEV_TIMEOUT and the caller is told; it then
// issues no further copy, drains what it issued (drain_stage) and reports
// that call's output invalid.  polls = 0 gives up at once unless the stage
// has already landed (the path a test takes to exercise the give-up).
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity, uint32_t *status,
                                                  uint32_t polls) {
    if (mbar_test_wait(bar, parity)) return true;
    for (uint32_t i = 0; i < polls; i++)
        if (mbar_try_wait(bar, parity)) return true;
    atomicOr(status, (uint32_t)KVQ_DEV_TIMEOUT);
    return false;
}

// ------------------------------------------------------------ launch set-up
// Raise a kernel's dynamic shared memory limit to `bytes` once per device and
// kernel instance, so that later launches (including those recorded into a
// CUDA graph) make no attribute calls.  `bytes` must be the instance's maximum.
template <typename Kernel>
cudaError_t set_smem_once(Kernel *fn, int bytes, std::atomic<uint64_t> &done) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = 1ull << (dev & 63);
    if (done.load(std::memory_order_acquire) & bit) return cudaSuccess;
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) done.fetch_or(bit, std::memory_order_release);
    return e;
}

// ------------------------------------------------------------ split merge
// Each CTA of a (sequence, KV head) unit writes one partial (running max m,
// sum l and output o per query head) for its split of the context.  The last
// CTA to arrive -- found with the unit's completion counter, which it resets
// -- merges them: out = sum_s e^{m_s - M} o_s / sum_s e^{m_s - M} l_s, the one
// softmax over the whole context (Dual-QK §3.4).  Nothing waits: the other
// CTAs simply exit.  Called by every thread of an NT-thread CTA; `scratch` is
// 16-byte aligned shared memory for merge_scratch_floats(G, NT, S) floats.
// The G * 128 outputs, as float4 columns, are summed over the splits with
// R = NT / columns threads per column (each a strided subset of the splits);
// the first kMergeChunk partials of every thread are loaded together with
// the (m, l) pairs, so the merge costs one round trip to L2 for S <= R *
// kMergeChunk, and the R partial sums are added in a fixed order.
// With a value rotation `rot` (the unit's KV head's 128 x 128 float64 matrix,
// row-major, 16-byte aligned; values were stored as V rot) the merged output
// is rotated back, out[c] = sum_j o[j] rot[c][j] (rot is orthogonal; §3.3
// reverses the value rotation after aggregation), in float64 over j
// ascending, in two halves added at the end when NT = 256.
template <int G, int NT>
struct MergeShape {
    static constexpr int F = G * kD / 4;                 // float4 columns
    static constexpr int R = NT >= F ? NT / F : 1;       // threads per column
    static constexpr int CPT = NT >= F ? 1 : F / NT;     // columns per thread
    static_assert(NT >= F ? NT % F == 0 : F % NT == 0, "merge: columns and threads must divide");
};
constexpr int kMergeChunk = 20;
__host__ __device__ constexpr int merge_scratch_floats(int G, int NT, int S) {
    return ((2 * G * S + G + 3) & ~3) + (NT > G * kD / 4 ? NT / (G * kD / 4) * G * kD : 0) + G * kD;
}
template <int G, int NT>
__device__ __forceinline__ void merge_unit_if_last(const float *part_o, const float2 *part_ml, int S,
                                                   size_t qrow0, float *out, uint32_t *counter,
                                                   float *scratch, const double *rot = nullptr) {
    using MS = MergeShape<G, NT>;
    static_assert(NT % kD == 0 && NT / kD <= 2, "rotation: one or two threads per output channel");
    __shared__ int s_last;
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        const unsigned prev = atomicAdd(counter, 1u);
        s_last = prev == (unsigned)S - 1u;
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    float *wm = scratch;             // [G][S] max, then weight
    float *wl = scratch + G * S;     // [G][S] sum
    float *inv = wl + G * S;         // [G] 1 / total sum
    float4 *part = reinterpret_cast<float4 *>(scratch + ((2 * G * S + G + 3) & ~3));   // [R][F]
    float *orot = reinterpret_cast<float *>(part) + (MS::R > 1 ? MS::R * MS::F * 4 : 0);   // [G][128]
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    // merged output of head hl, channels c0..c0+3: to `out`, or to shared
    // memory when it is still to be rotated back
    auto emit = [&](int hl, int c0, float4 a) {
        float *o = rot ? orot + hl * kD + c0 : out + (qrow0 + hl) * kD + c0;   // out is only 4-byte aligned
        o[0] = a.x;
        o[1] = a.y;
        o[2] = a.z;
        o[3] = a.w;
    };
    const int sub = t / (NT / MS::R >= 1 ? NT / MS::R : 1);   // split subset of this thread
    const int col0 = (t % (NT / MS::R)) * MS::CPT;
    auto column = [&](int col) {
        const int hl = (4 * col) / kD, c0 = (4 * col) % kD;
        return reinterpret_cast<const float4 *>(part_o + ((qrow0 + hl) * S) * kD + c0);
    };
    // the first chunk of the first column's partials, in flight with the (m, l) pass
    float4 v[kMergeChunk];
    {
        const float4 *po = column(col0);
#pragma unroll
        for (int j = 0; j < kMergeChunk; j++) {
            const int sj = sub + j * MS::R;
            v[j] = sj < S ? __ldcg(po + (size_t)sj * (kD / 4)) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
    for (int e = t; e < G * S; e += NT) {
        const float2 ml = __ldcg(part_ml + qrow0 * S + e);     // rows qrow0.. are contiguous
        wm[e] = ml.x;
        wl[e] = ml.y;
    }
    __syncthreads();
    for (int hl = warp; hl < G; hl += NT / 32) {
        float M = -INFINITY;
        for (int s = lane; s < S; s += 32) M = fmaxf(M, wm[hl * S + s]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
        float L = 0.f;
        for (int s = lane; s < S; s += 32) {
            const float w = (M == -INFINITY) ? 0.f : exp2f(wm[hl * S + s] - M);
            wm[hl * S + s] = w;
            L = fmaf(w, wl[hl * S + s], L);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
        if (lane == 0) inv[hl] = L > 0.f ? 1.f / L : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int cc = 0; cc < MS::CPT; cc++) {
        const int col = col0 + cc, hl = (4 * col) / kD, c0 = (4 * col) % kD;
        const float4 *po = column(col);
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int j0 = 0; sub + j0 * MS::R < S; j0 += kMergeChunk) {
            if (cc > 0 || j0 > 0) {
#pragma unroll
                for (int j = 0; j < kMergeChunk; j++) {
                    const int sj = sub + (j0 + j) * MS::R;
                    v[j] = sj < S ? __ldcg(po + (size_t)sj * (kD / 4)) : make_float4(0.f, 0.f, 0.f, 0.f);
                }
            }
#pragma unroll
            for (int j = 0; j < kMergeChunk; j++) {
                const int sj = sub + (j0 + j) * MS::R;
                const float w = sj < S ? wm[hl * S + sj] : 0.f;
                acc.x = fmaf(w, v[j].x, acc.x);
                acc.y = fmaf(w, v[j].y, acc.y);
                acc.z = fmaf(w, v[j].z, acc.z);
                acc.w = fmaf(w, v[j].w, acc.w);
            }
        }
        if constexpr (MS::R == 1) {
            const float r = inv[hl];
            emit(hl, c0, make_float4(acc.x * r, acc.y * r, acc.z * r, acc.w * r));
        } else {
            part[sub * MS::F + col] = acc;
        }
    }
    if constexpr (MS::R > 1) {
        __syncthreads();
        for (int col = t; col < MS::F; col += NT) {
            const int hl = (4 * col) / kD, c0 = (4 * col) % kD;
            float4 a = part[col];
            for (int q = 1; q < MS::R; q++) {
                const float4 v2 = part[q * MS::F + col];
                a.x += v2.x; a.y += v2.y; a.z += v2.z; a.w += v2.w;
            }
            const float r = inv[hl];
            emit(hl, c0, make_float4(a.x * r, a.y * r, a.z * r, a.w * r));
        }
    }
    if (rot) {
        __syncthreads();
        constexpr int P = NT / kD;                       // threads per output channel
        constexpr int J = kD / P;                        // terms per thread
        const int c = t / P, j0 = (t % P) * J;
        const double2 *row = reinterpret_cast<const double2 *>(rot + (size_t)c * kD + j0);
        double acc[G];
#pragma unroll
        for (int hl = 0; hl < G; hl++) acc[hl] = 0.0;
#pragma unroll 8
        for (int jj = 0; jj < J / 2; jj++) {
            const double2 r2 = __ldg(row + jj);
#pragma unroll
            for (int hl = 0; hl < G; hl++) {
                acc[hl] = fma((double)orot[hl * kD + j0 + 2 * jj], r2.x, acc[hl]);
                acc[hl] = fma((double)orot[hl * kD + j0 + 2 * jj + 1], r2.y, acc[hl]);
            }
        }
#pragma unroll
        for (int hl = 0; hl < G; hl++) {
            if constexpr (P == 2) acc[hl] += __shfl_xor_sync(0xffffffffu, acc[hl], 1);
            if (t % P == 0) out[(qrow0 + hl) * kD + c] = (float)acc[hl];
        }
    }
    __syncthreads();
    if (t == 0) atomicExch(counter, 0u);
}

// ------------------------------------------------------------ protected tier partial
// The protected tier's share of one unit's softmax (Dual-QK §3.3: BF16 keys
// and values, the same query-channel mask; §3.4: one softmax over all tiers),
// for the unit's slots [slot0, slot1): scores of the G query heads over the
// selected channels (1/sqrt(128), base-2 exponent domain like the codes'
// scores), an online softmax over chunks of kTierChunk slots, value
// aggregation, written as split s of the unit's partials (m, l, o).  Slots
// that hold no protected position of a sequence of length len count as empty.
// Called by every thread of an NT-thread CTA; q'[head hl] of list position i
// is q[hl * hs + i * ps], `chan` the channel list, both in shared memory;
// `scratch` is shared memory of tier_scratch_floats(G) floats.
constexpr int kTierChunk = 32;
__host__ __device__ constexpr int tier_scratch_floats(int G) {
    return kD * (kTierChunk + 1) + kTierChunk * kD + G * kTierChunk + 4 * G;
}
// Where the tier's scores take the query coefficients and the channel list
// of a protected position p: one selection in shared memory (q'[head hl] of
// list position i at q[hl * hs + i * ps]), or -- with RoPE buckets -- the
// selection arrays of p's bucket in global memory (list entries clamped into
// 0..127).
struct TierQShared {
    const float *q;
    int hs, ps;
    const int *chan;
    __device__ float q_at(int hl, int i, int) const { return q[hl * hs + i * ps]; }
    __device__ int ch(int i, int) const { return chan[i]; }
};
struct TierQBuckets {
    const float *qsel;             // [..][nb][k] rows of this unit's heads from qrow0
    const int32_t *idx;            // [nb][k] of this unit
    int k, nb, w;
    size_t qrow0;
    __device__ float q_at(int hl, int i, int p) const { return __ldg(qsel + ((qrow0 + hl) * nb + p / w) * k + i); }
    __device__ int ch(int i, int p) const { return min(max(__ldg(idx + (size_t)(p / w) * k + i), 0), kD - 1); }
};
template <int G, int NT, typename QS>
__device__ void tier_partial(const uint8_t *__restrict__ slots, int len, int n_sink, int n_recent, int slot0,
                             int slot1, const QS &qs, int k,
                             float *__restrict__ part_o, float2 *__restrict__ part_ml, size_t qrow0, int S, int s,
                             float *scratch) {
    constexpr int C = kTierChunk;
    constexpr int OPT = G * kD / NT;                   // outputs per thread, all of one head
    static_assert(OPT >= 1 && OPT * NT == G * kD && kD % OPT == 0, "tier: outputs must divide the threads");
    float *kT = scratch;                               // [128][C + 1] keys, channel-major
    float *vv = kT + kD * (C + 1);                     // [C][128] values
    float *sc = vv + C * kD;                           // [G][C] scores, then weights
    float *m_run = sc + G * C;                         // [G]
    float *m_use = m_run + G;                          // [G]
    float *alpha = m_use + G;                          // [G]
    float *l_run = alpha + G;                          // [G]
    const Tier tr = tier_of(len, n_sink, n_recent);
    const int t = threadIdx.x;
    const int oh = (t * OPT) / kD, oc = (t * OPT) % kD;
    float o[OPT];
#pragma unroll
    for (int u = 0; u < OPT; u++) o[u] = 0.f;
    if (t < G) {
        m_run[t] = -INFINITY;
        l_run[t] = 0.f;
    }
    for (int c0 = slot0; c0 < slot1; c0 += C) {
        const int n = min(C, slot1 - c0);
        __syncthreads();                               // the previous chunk is consumed
        for (int e = t; e < C * (kD / 2); e += NT) {
            const int tt = e / (kD / 2), cp = e % (kD / 2);
            uint32_t kw = 0, vw = 0;
            if (tt < n) {
                const uint32_t *row = reinterpret_cast<const uint32_t *>(slots + (size_t)(c0 + tt) * kSlotBytes);
                kw = __ldg(row + cp);
                vw = __ldg(row + kD / 2 + cp);
            }
            kT[(2 * cp) * (C + 1) + tt] = __uint_as_float(kw << 16);
            kT[(2 * cp + 1) * (C + 1) + tt] = __uint_as_float(kw & 0xffff0000u);
            vv[tt * kD + 2 * cp] = __uint_as_float(vw << 16);
            vv[tt * kD + 2 * cp + 1] = __uint_as_float(vw & 0xffff0000u);
        }
        __syncthreads();
        for (int e = t; e < G * C; e += NT) {
            const int hl = e / C, tt = e % C, slot = c0 + tt;
            bool valid = false;
            int p = slot;                              // the position this slot holds
            if (tt < n) {
                if (slot < n_sink) {
                    valid = slot < tr.sink_end;
                } else if (n_recent > 0) {
                    // the one position of the recent window that owns this ring slot
                    const int j = slot - n_sink;
                    p = tr.recent_start + ((j - tr.recent_start % n_recent) % n_recent + n_recent) % n_recent;
                    valid = p < len;
                }
            }
            float v = -INFINITY;
            if (valid) {
                float a = 0.f;
                for (int i = 0; i < k; i++) a = fmaf(qs.q_at(hl, i, p), kT[qs.ch(i, p) * (C + 1) + tt], a);
                v = a * kScoreScaleLog2;
            }
            sc[e] = v;
        }
        __syncthreads();
        if (t < G) {
            float m = m_run[t];
            for (int tt = 0; tt < C; tt++) m = fmaxf(m, sc[t * C + tt]);
            const float mu = (m == -INFINITY) ? 0.f : m;
            alpha[t] = exp2f(m_run[t] - mu);
            m_use[t] = mu;
            m_run[t] = m;
        }
        __syncthreads();
        for (int e = t; e < G * C; e += NT) sc[e] = exp2f(sc[e] - m_use[e / C]);
        __syncthreads();
        if (t < G) {
            float ls = 0.f;
            for (int tt = 0; tt < C; tt++) ls += sc[t * C + tt];
            l_run[t] = fmaf(l_run[t], alpha[t], ls);
        }
        const float a = alpha[oh];
#pragma unroll
        for (int u = 0; u < OPT; u++) o[u] *= a;
        for (int tt = 0; tt < n; tt++) {
            const float p = sc[oh * C + tt];
#pragma unroll
            for (int u = 0; u < OPT; u++) o[u] = fmaf(p, vv[tt * kD + oc + u], o[u]);
        }
    }
    __syncthreads();
    const size_t row = (qrow0 + oh) * S + s;
#pragma unroll
    for (int u = 0; u < OPT; u++) part_o[row * kD + oc + u] = o[u];
    if (oc == 0) part_ml[row] = make_float2(m_run[oh], l_run[oh]);
}

}  // namespace kvq

// launchers implemented in the .cu files (host side, called by kvq_api.cu)
namespace kvq {
cudaError_t launch_append(const kvq_cache &c, const void *K, const void *V, int dtype, int n_new,
                          const double *A, cudaStream_t st);
cudaError_t launch_select(const kvq_cache &c, const void *q, int dtype, int Hq, const double *Ainvt,
                          const double *delta, int k, int32_t *idx, float *qsel, float *qgsum, cudaStream_t st);
int decode_splits(const kvq_cache &c, int Hq, int k, int num_sms);
size_t decode_ws_bytes(const kvq_cache &c, int Hq, int n_splits, bool step = false);
cudaError_t launch_decode(const kvq_cache &c, int Hq, const int32_t *idx, const float *qsel,
                          const float *qgsum, int k, float *out, void *ws, int n_splits,
                          cudaStream_t st, long long polls = -1);
bool decode_uses_mma(const kvq_cache &c, int Hq);
cudaError_t launch_decode_step(const kvq_cache &c, int Hq, const void *q, const void *k_new,
                               const void *v_new, int dtype, int n_new, const double *A,
                               const double *Ainvt, const double *delta, int k, int32_t *idx, float *qsel,
                               float *qgsum, float *out, void *ws, int n_splits, cudaStream_t st);
// completion counter of unit (b, h) in the cache's status array
inline uint32_t *unit_counter(const kvq_cache &c, int b, int h) {
    return c.status + 1 + c.batch + (size_t)b * c.n_kv_heads + h;
}
int bf16_splits(int B, int Hkv, int N, int num_sms);
size_t bf16_ws_bytes(int B, int Hq, int n_splits);
cudaError_t launch_bf16_decode(const void *q, const void *K, const void *V, int B, int Hq, int Hkv,
                               int N, float *out, void *ws, int n_splits, cudaStream_t st);
}  // namespace kvq
