// Unpruned, unquantized BF16 decode attention: the comparator the Dual-QK
// pages measure against ("unpruned BF16", §4.4), plain softmax(q K^T /
// sqrt(128)) V over every token, split over the context with the same exact
// merge as the quantized path.
//
// It reads 512 bytes per token and KV head and computes little, so the design
// is about keeping enough bytes in flight: one CTA = one (sequence, KV head,
// split), four warps, a ring of three stages of 64-token K and V tiles filled
// by one 256-byte bulk asynchronous copy per row (rows padded to 272 bytes,
// which makes every fragment load below bank-conflict free), each stage's
// copies completing on an mbarrier that all 128 threads arrive on with the
// bytes of their own row.  Warp w takes tokens 16w..16w+15 of every tile, on
// the tensor cores (mma.sync m16n8k16, bf16 in, f32 accumulate):
//   scores S[head][token] = q[head][channel] . K^T[channel][token]
//     (the query heads are the M rows, padded to 16), whose C fragment is
//     exactly the B fragment of
//   out^T[channel][head] += V^T[channel][token] . P[token][head]
//     (V^T fragments by ldmatrix.trans from the token-major rows),
// with the softmax weights as bf16 hi + lo pairs in the value MMAs (the
// values are exact bf16, the weights keep about 16 bits) and an online
// softmax per warp, merged over the warps at the end.
#include "kvq_internal.cuh"

namespace kvq {
namespace {

constexpr int kTT = 64;                        // tokens per tile
constexpr int kThr = 128;                      // 4 warps x 16 tokens
constexpr int kStagesB = 3;
constexpr int kRowPad = 2 * kD + 16;           // bytes per staged row (padded)
constexpr int kTileB = kTT * kRowPad;          // one staged K or V tile
constexpr uint32_t kPollsB = 1u << 20;         // bound on mbarrier polls per stage

struct __align__(16) Bf16Shared {
    uint8_t k[kStagesB][kTileB];
    uint8_t v[kStagesB][kTileB];
    uint64_t full[kStagesB];
};

__device__ __forceinline__ uint32_t smem_u32b(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                              uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;\n" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}
__device__ __forceinline__ float ex2b(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
    return y;
}

// One row (token) of a tile into its stage: the thread's share of the
// stage's expected bytes, then the copy (nothing for a token past the end).
__device__ __forceinline__ void stage_row(uint8_t *dst, const uint16_t *src, bool valid, uint32_t bar) {
    const uint32_t bytes = valid ? 2u * kD : 0u;
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(bar), "r"(bytes) : "memory");
    if (valid)
        asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n"
                     ::"r"(smem_u32b(dst)), "l"(src), "r"(bytes), "r"(bar) : "memory");
}
__device__ __forceinline__ bool wait_stage(uint32_t bar, uint32_t parity) {
    for (uint32_t i = 0; i < kPollsB; i++) {
        uint32_t ok;
        asm volatile(
            "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
            : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
        if (ok) return true;
    }
    return false;
}

template <int G>
__global__ void __launch_bounds__(kThr, 2)
bf16_decode_kernel(const uint16_t *__restrict__ q, const uint16_t *__restrict__ K,
                   const uint16_t *__restrict__ V, int Hq, int Hkv, int N,
                   float *__restrict__ part_o, float2 *__restrict__ part_ml, int S) {
    static_assert(G >= 1 && G <= 8, "heads per KV head: the 8 columns of the value MMA");
    extern __shared__ __align__(16) uint8_t smem_raw[];
    Bf16Shared &sh = *reinterpret_cast<Bf16Shared *>(smem_raw);

    const int s = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int gid = lane >> 2, tig = lane & 3;
    const size_t unit = (size_t)b * Hkv + h;
    const uint16_t *Kb = K + unit * (size_t)N * kD;
    const uint16_t *Vb = V + unit * (size_t)N * kD;
    const size_t qrow0 = (size_t)b * Hq + (size_t)h * G;

    const int ntile = (N + kTT - 1) / kTT;
    const int tps = (ntile + S - 1) / S;
    const int tile0 = min(ntile, s * tps), tile1 = min(ntile, tile0 + tps);

    if (tid < kStagesB) asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_u32b(&sh.full[tid])), "r"(kThr) : "memory");
    // stale rows are multiplied by zero weights: start from finite bytes
    for (int e = tid; e < (int)(sizeof(sh.k) + sizeof(sh.v)) / 16; e += kThr)
        reinterpret_cast<uint4 *>(&sh.k[0][0])[e] = make_uint4(0, 0, 0, 0);
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
    __syncthreads();

    // thread t stages row t % 64 of K (t < 64) or of V (t >= 64)
    auto issue = [&](int tile, int st) {
        const int row = tid & (kTT - 1), tok = tile * kTT + row;
        const bool valid = tok < N;
        const size_t src = (size_t)(valid ? tok : 0) * kD;
        if (tid < kTT) stage_row(sh.k[st] + row * kRowPad, Kb + src, valid, smem_u32b(&sh.full[st]));
        else stage_row(sh.v[st] + row * kRowPad, Vb + src, valid, smem_u32b(&sh.full[st]));
    };
    for (int i = 0; i < kStagesB && tile0 + i < tile1; i++) issue(tile0 + i, i);

    // query fragments (rows = heads gid < G, channels 16ks + 2tig (+8)), bf16 pairs
    uint32_t qa[8][2];
#pragma unroll
    for (int ks = 0; ks < 8; ks++) {
#pragma unroll
        for (int hf = 0; hf < 2; hf++) {
            uint32_t w = 0;
            if (gid < G)
                w = *reinterpret_cast<const uint32_t *>(q + (qrow0 + gid) * kD + 16 * ks + 2 * tig + 8 * hf);
            qa[ks][hf] = w;
        }
    }

    float m_run = -INFINITY;        // running max of head gid (base-2 domain)
    float l_thr = 0.f;              // this thread's share of head gid's sum
    float o[8][4];                  // out^T: m-tile mt, rows channel 16mt+gid (+8), cols heads 2tig (+1)
#pragma unroll
    for (int mt = 0; mt < 8; mt++)
#pragma unroll
        for (int r = 0; r < 4; r++) o[mt][r] = 0.f;

    int stop = tile1;                  // a wait that gives up ends the loop there
    for (int tile = tile0; tile < tile1; tile++) {
        const int it = tile - tile0, st = it % kStagesB;
        const uint32_t par = (uint32_t)(it / kStagesB) & 1u;
        if (!__syncthreads_and(wait_stage(smem_u32b(&sh.full[st]), par))) {
            stop = tile;
            break;
        }
        const uint8_t *kst = sh.k[st] + (16 * warp) * kRowPad;
        const uint8_t *vst = sh.v[st] + (16 * warp) * kRowPad;

        // scores of this warp's 16 tokens: n-tile j = tokens 8j..8j+7
        float c[2][4];
#pragma unroll
        for (int j = 0; j < 2; j++) {
#pragma unroll
            for (int r = 0; r < 4; r++) c[j][r] = 0.f;
            const uint8_t *kr = kst + (8 * j + gid) * kRowPad + 4 * tig;
#pragma unroll
            for (int ks = 0; ks < 8; ks++) {
                const uint32_t b0 = *reinterpret_cast<const uint32_t *>(kr + 32 * ks);
                const uint32_t b1 = *reinterpret_cast<const uint32_t *>(kr + 32 * ks + 16);
                mma_bf16(c[j], qa[ks][0], 0u, qa[ks][1], 0u, b0, b1);
            }
        }
        // head gid, tokens 16w + 8j + 2tig + r: base-2 scores, masked past the end
        const int tbase = tile * kTT + 16 * warp;
        float sc[2][2];
        float mx = -INFINITY;
#pragma unroll
        for (int j = 0; j < 2; j++)
#pragma unroll
            for (int r = 0; r < 2; r++) {
                const int tok = tbase + 8 * j + 2 * tig + r;
                sc[j][r] = tok < N ? c[j][r] * kScoreScaleLog2 : -INFINITY;
                mx = fmaxf(mx, sc[j][r]);
            }
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        const float m_new = fmaxf(m_run, mx);
        const float m_use = m_new == -INFINITY ? 0.f : m_new;
        const float alpha = ex2b(m_run - m_use);
        m_run = m_new;
        float p[2][2];
        l_thr *= alpha;
#pragma unroll
        for (int j = 0; j < 2; j++)
#pragma unroll
            for (int r = 0; r < 2; r++) {
                p[j][r] = ex2b(sc[j][r] - m_use);
                l_thr += p[j][r];
            }
        // the C fragment of the scores is the B fragment of the weights:
        // k = tokens 2tig, 2tig+1 (+8), n = head gid; each weight as a bf16
        // hi + lo pair (about 16 significant bits, two MMAs) so that the
        // weights' rounding stays far below the output tolerance
        uint32_t ph[2], pl[2];
#pragma unroll
        for (int j = 0; j < 2; j++) {
            ph[j] = pack_bf16(p[j][0], p[j][1]);
            const float h0 = __uint_as_float(ph[j] << 16), h1 = __uint_as_float(ph[j] & 0xffff0000u);
            pl[j] = pack_bf16(p[j][0] - h0, p[j][1] - h1);
        }
        // rescale: out^T column 2tig + r is head 2tig + r, whose alpha lane 4(2tig + r) holds
        const float a0 = __shfl_sync(0xffffffffu, alpha, 8 * tig);
        const float a1 = __shfl_sync(0xffffffffu, alpha, 8 * tig + 4);
        if (!__all_sync(0xffffffffu, a0 == 1.f && a1 == 1.f)) {
#pragma unroll
            for (int mt = 0; mt < 8; mt++) {
                o[mt][0] *= a0; o[mt][1] *= a1; o[mt][2] *= a0; o[mt][3] *= a1;
            }
        }
        // values: m-tile mt = channels 16mt..16mt+15, k = the warp's 16 tokens
        {
            const int mi = lane >> 3, rr = lane & 7;
            const uint32_t vaddr = smem_u32b(vst + (rr + 8 * (mi >> 1)) * kRowPad + 16 * (mi & 1));
#pragma unroll
            for (int mt = 0; mt < 8; mt++) {
                uint32_t a0r, a1r, a2r, a3r;
                ldsm_x4_trans(vaddr + 32 * mt, a0r, a1r, a2r, a3r);
                mma_bf16(o[mt], a0r, a1r, a2r, a3r, ph[0], ph[1]);
                mma_bf16(o[mt], a0r, a1r, a2r, a3r, pl[0], pl[1]);
            }
        }
        __syncthreads();                               // every warp is done with stage st
        if (tile + kStagesB < tile1) issue(tile + kStagesB, st);
    }
    if (stop < tile1) {
        // the stages still in flight land before the memory is reused; the
        // partial is written as NaN so that the result shows it
        for (int tile = stop; tile < min(tile1, stop + kStagesB); tile++) {
            const int it = tile - tile0;
            wait_stage(smem_u32b(&sh.full[it % kStagesB]), (uint32_t)(it / kStagesB) & 1u);
        }
        m_run = __int_as_float(0x7fc00000);
    }

    // merge the 4 warps: per head max and sum, then the outputs
    __syncthreads();
    float *mo = reinterpret_cast<float *>(&sh.k[0][0]);          // [warp][head 8][128]
    float *mml = mo + 4 * 8 * kD;                                // [warp][head 8][2]
    float l_head = l_thr;
    l_head += __shfl_xor_sync(0xffffffffu, l_head, 1);
    l_head += __shfl_xor_sync(0xffffffffu, l_head, 2);
    if (tig == 0) {
        mml[(warp * 8 + gid) * 2] = m_run;
        mml[(warp * 8 + gid) * 2 + 1] = l_head;
    }
#pragma unroll
    for (int mt = 0; mt < 8; mt++) {
        const int ch = 16 * mt + gid;
        mo[(warp * 8 + 2 * tig) * kD + ch] = o[mt][0];
        mo[(warp * 8 + 2 * tig + 1) * kD + ch] = o[mt][1];
        mo[(warp * 8 + 2 * tig) * kD + ch + 8] = o[mt][2];
        mo[(warp * 8 + 2 * tig + 1) * kD + ch + 8] = o[mt][3];
    }
    __syncthreads();
    for (int e = tid; e < G * kD; e += kThr) {
        const int hl = e / kD, ch = e % kD;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < 4; w++) M = fmaxf(M, mml[(w * 8 + hl) * 2]);
        float ov = 0.f, L = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < 4; w++) {
                const float wt = exp2f(mml[(w * 8 + hl) * 2] - M);
                L = fmaf(wt, mml[(w * 8 + hl) * 2 + 1], L);
                ov = fmaf(wt, mo[(w * 8 + hl) * kD + ch], ov);
            }
        }
        const size_t row = (qrow0 + hl) * S + s;
        part_o[row * kD + ch] = ov;
        if (ch == 0) part_ml[row] = make_float2(M, L);
    }
}

template <int G>
cudaError_t launch_bf16_t(const void *q, const void *K, const void *V, int B, int Hq, int Hkv, int N,
                          float *part_o, float2 *part_ml, int S, cudaStream_t st) {
    static_assert(sizeof(Bf16Shared) >= (4 * 8 * kD + 4 * 8 * 2) * sizeof(float), "merge scratch fits the stages");
    const size_t smem = sizeof(Bf16Shared);
    auto fn = bf16_decode_kernel<G>;
    static std::atomic<uint64_t> done{0};
    cudaError_t e = set_smem_once(fn, (int)smem, done);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)S, (unsigned)Hkv, (unsigned)B);
    fn<<<grid, kThr, smem, st>>>(static_cast<const uint16_t *>(q), static_cast<const uint16_t *>(K),
                                 static_cast<const uint16_t *>(V), Hq, Hkv, N, part_o, part_ml, S);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_combine(int rows, const float *part_o, const float2 *part_ml, int S, float *out,
                           cudaStream_t st);

int bf16_splits(int B, int Hkv, int N, int num_sms) {
    const int units = B * Hkv;
    const int ntile = (N + kTT - 1) / kTT;
    int S = (2 * num_sms) / units;                      // about two CTAs per SM
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
