// Unpruned, unquantized BF16 decode attention: the comparator the Dual-QK
// pages measure against ("unpruned BF16", §4.4).  Same split-over-context
// structure and merge as the quantized path.
//
// One CTA = one (sequence, KV head, split), 128 threads, 64-token tiles of K
// and V staged with cp.async (double buffered; key rows stored with their
// 16-byte chunks XOR-swizzled by row so that per-token 16-byte reads are
// bank-conflict free).  Scores: two threads per token, 64 channels each.
// Values: each thread owns two channels and half of the tile's tokens.
#include "kvq_internal.cuh"

namespace kvq {
namespace {

constexpr int kTT = 64;                       // tokens per tile
constexpr int kTileBytes = kTT * kD * 2;      // one K or V tile

__device__ __forceinline__ void cp_async16_zfill(void *smem_dst, const void *gmem_src, bool valid) {
    uint32_t d = (uint32_t)__cvta_generic_to_shared(smem_dst);
    int n = valid ? 16 : 0;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(d), "l"(gmem_src), "r"(n)
                 : "memory");
}

__device__ __forceinline__ float warp_max_f(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

template <int G>
__global__ void __launch_bounds__(128)
bf16_decode_kernel(const uint16_t *__restrict__ q, const uint16_t *__restrict__ K,
                   const uint16_t *__restrict__ V, int Hq, int Hkv, int N,
                   float *__restrict__ part_o, float2 *__restrict__ part_ml, int S) {
    extern __shared__ __align__(16) uint8_t smem[];
    uint8_t *kst[2] = {smem, smem + 2 * kTileBytes};
    uint8_t *vst[2] = {smem + kTileBytes, smem + 3 * kTileBytes};
    float *sq = reinterpret_cast<float *>(smem + 4 * kTileBytes);   // [G][128]
    float *ss = sq + G * kD;                                          // [2][64][G]
    float *sp = ss + 2 * kTT * G;                                     // [64][G]
    float *sred = sp + kTT * G;                                       // [2][G]
    float *sfin = sred + 2 * G;                                       // [G][128] + [G]

    const int s = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const size_t unit = (size_t)b * Hkv + h;
    const uint16_t *Kb = K + unit * (size_t)N * kD;
    const uint16_t *Vb = V + unit * (size_t)N * kD;

    for (int e = tid; e < G * kD; e += 128)
        sq[e] = __uint_as_float(((uint32_t)q[((size_t)b * Hq + (size_t)h * G) * kD + e]) << 16);

    const int ntile = (N + kTT - 1) / kTT;
    const int tps = (ntile + S - 1) / S;
    const int tile0 = s * tps, tile1 = min(ntile, tile0 + tps);

    auto load = [&](int st, int tile) {
        for (int e = tid; e < kTT * 16; e += 128) {
            const int row = e >> 4, ch = e & 15;
            const int tok = tile * kTT + row;
            const bool ok = tok < N;
            const size_t src = (size_t)(ok ? tok : 0) * kD + ch * 8;
            cp_async16_zfill(kst[st] + row * 256 + ((ch ^ (row & 7)) * 16), Kb + src, ok);
            cp_async16_zfill(vst[st] + row * 256 + ch * 16, Vb + src, ok);
        }
        cp_async_commit();
    };

    float m_run[G], l_run[G], o0[G], o1[G];
#pragma unroll
    for (int hl = 0; hl < G; hl++) {
        m_run[hl] = -INFINITY;
        l_run[hl] = 0.f;
        o0[hl] = 0.f;
        o1[hl] = 0.f;
    }
    __syncthreads();

    if (tile0 < tile1) load(0, tile0);
    for (int tile = tile0; tile < tile1; tile++) {
        const int st = (tile - tile0) & 1;
        if (tile + 1 < tile1) {
            load(st ^ 1, tile + 1);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();

        // scores: token tid&63, channel half tid>>6
        {
            const int tok = tid & (kTT - 1), half = tid >> 6;
            float acc[G];
#pragma unroll
            for (int hl = 0; hl < G; hl++) acc[hl] = 0.f;
#pragma unroll
            for (int cc = 0; cc < 8; cc++) {
                const int ch = half * 8 + cc;
                const uint4 w = *reinterpret_cast<const uint4 *>(kst[st] + tok * 256 + ((ch ^ (tok & 7)) * 16));
                const float kf[8] = {bf_lo(w.x), bf_hi(w.x), bf_lo(w.y), bf_hi(w.y),
                                     bf_lo(w.z), bf_hi(w.z), bf_lo(w.w), bf_hi(w.w)};
#pragma unroll
                for (int e = 0; e < 8; e++)
#pragma unroll
                    for (int hl = 0; hl < G; hl++) acc[hl] = fmaf(sq[hl * kD + ch * 8 + e], kf[e], acc[hl]);
            }
#pragma unroll
            for (int hl = 0; hl < G; hl++) ss[(half * kTT + tok) * G + hl] = acc[hl];
        }
        __syncthreads();
        float sc[G];
#pragma unroll
        for (int hl = 0; hl < G; hl++) sc[hl] = -INFINITY;
        if (tid < kTT) {
            const bool valid = tile * kTT + tid < N;
#pragma unroll
            for (int hl = 0; hl < G; hl++) {
                const float v = (ss[tid * G + hl] + ss[(kTT + tid) * G + hl]) * kScoreScaleLog2;
                sc[hl] = valid ? v : -INFINITY;
                const float wm = warp_max_f(sc[hl]);
                if (lane == 0) sred[warp * G + hl] = wm;
            }
        }
        __syncthreads();
#pragma unroll
        for (int hl = 0; hl < G; hl++) {
            const float mn = fmaxf(m_run[hl], fmaxf(sred[hl], sred[G + hl]));
            const float alpha = exp2f(m_run[hl] - mn);
            m_run[hl] = mn;
            l_run[hl] *= alpha;
            o0[hl] *= alpha;
            o1[hl] *= alpha;
            if (tid < kTT) sp[tid * G + hl] = exp2f(sc[hl] - mn);
        }
        __syncthreads();

        // values: channel pair tid&63, token half tid>>6
        {
            const int cp = tid & 63, th = tid >> 6;
#pragma unroll 4
            for (int t = th * 32; t < th * 32 + 32; t++) {
                const uint32_t w = *reinterpret_cast<const uint32_t *>(vst[st] + t * 256 + cp * 4);
                const float v0 = bf_lo(w), v1 = bf_hi(w);
#pragma unroll
                for (int hl = 0; hl < G; hl++) {
                    const float p = sp[t * G + hl];
                    o0[hl] = fmaf(p, v0, o0[hl]);
                    o1[hl] = fmaf(p, v1, o1[hl]);
                    l_run[hl] += p;
                }
            }
        }
        __syncthreads();
    }

    // merge the two token halves and write this split's partial
    const int cp = tid & 63, th = tid >> 6;
    if (th == 1) {
#pragma unroll
        for (int hl = 0; hl < G; hl++) {
            sfin[hl * kD + 2 * cp] = o0[hl];
            sfin[hl * kD + 2 * cp + 1] = o1[hl];
            if (cp == 0) sfin[G * kD + hl] = l_run[hl];
        }
    }
    __syncthreads();
    if (th == 0) {
#pragma unroll
        for (int hl = 0; hl < G; hl++) {
            const size_t row = ((size_t)b * Hq + (size_t)h * G + hl) * S + s;
            part_o[row * kD + 2 * cp] = o0[hl] + sfin[hl * kD + 2 * cp];
            part_o[row * kD + 2 * cp + 1] = o1[hl] + sfin[hl * kD + 2 * cp + 1];
            if (cp == 0) part_ml[row] = make_float2(m_run[hl], l_run[hl] + sfin[G * kD + hl]);
        }
    }
}

template <int G>
cudaError_t launch_bf16_t(const void *q, const void *K, const void *V, int B, int Hq, int Hkv, int N,
                          float *part_o, float2 *part_ml, int S, cudaStream_t st) {
    const size_t smem = 4 * (size_t)kTileBytes + sizeof(float) * (G * kD + 2 * kTT * G + kTT * G + 2 * G + G * kD + G);
    auto fn = bf16_decode_kernel<G>;
    static std::atomic<uint64_t> done{0};
    cudaError_t e = set_smem_once(fn, (int)smem, done);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)S, (unsigned)Hkv, (unsigned)B);
    fn<<<grid, 128, smem, st>>>(static_cast<const uint16_t *>(q), static_cast<const uint16_t *>(K),
                                static_cast<const uint16_t *>(V), Hq, Hkv, N, part_o, part_ml, S);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_combine(int rows, const float *part_o, const float2 *part_ml, int S, float *out,
                           cudaStream_t st);

int bf16_splits(int B, int Hkv, int N, int num_sms) {
    const int units = B * Hkv;
    const int ntile = (N + kTT - 1) / kTT;
    int S = (2 * num_sms + units - 1) / units;          // about two CTAs per SM
    S = S < 1 ? 1 : S;
    const int max_s = (ntile + 1) / 2 > 0 ? (ntile + 1) / 2 : 1;   // >= 2 tiles per split
    return S > max_s ? max_s : S;
}

size_t bf16_ws_bytes(int B, int Hq, int S) {
    return (size_t)B * Hq * S * (kD * sizeof(float) + sizeof(float2));
}

cudaError_t launch_bf16_decode(const void *q, const void *K, const void *V, int B, int Hq, int Hkv,
                               int N, float *out, void *ws, int S, cudaStream_t st) {
    float *part_o = static_cast<float *>(ws);
    float2 *part_ml = reinterpret_cast<float2 *>(part_o + (size_t)B * Hq * S * kD);
    const int g = Hq / Hkv;
    cudaError_t e;
    switch (g) {
        case 1: e = launch_bf16_t<1>(q, K, V, B, Hq, Hkv, N, part_o, part_ml, S, st); break;
        case 2: e = launch_bf16_t<2>(q, K, V, B, Hq, Hkv, N, part_o, part_ml, S, st); break;
        case 4: e = launch_bf16_t<4>(q, K, V, B, Hq, Hkv, N, part_o, part_ml, S, st); break;
        case 8: e = launch_bf16_t<8>(q, K, V, B, Hq, Hkv, N, part_o, part_ml, S, st); break;
        default: return cudaErrorInvalidValue;
    }
    if (e != cudaSuccess) return e;
    return launch_combine(B * Hq, part_o, part_ml, S, out, st);
}

}  // namespace kvq
