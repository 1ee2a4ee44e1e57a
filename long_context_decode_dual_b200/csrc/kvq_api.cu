// C ABI entry points (include/kvq.h): host-side validation, then launches.
#include <math.h>

#include "kvq_internal.cuh"

using namespace kvq;

namespace {

bool aligned(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }

int check_cache(const kvq_cache *c) {
    if (!c || !c->pages || !c->seq_len || !c->status) return KVQ_ERR_ARG;
    if (c->batch < 1 || c->n_kv_heads < 1 || c->capacity < 1) return KVQ_ERR_ARG;
    if (c->head_dim != kD || (c->group != kGroup && c->group != kD) || (c->bits != 2 && c->bits != 4))
        return KVQ_ERR_SHAPE;
    if (c->capacity % kT) return KVQ_ERR_SHAPE;
    if (c->n_sink < 0 || c->n_recent < 0 || c->n_sink + c->n_recent > KVQ_MAX_PROTECTED) return KVQ_ERR_ARG;
    if (!(c->v_clip == 0.0 || (c->v_clip > 0.0 && c->v_clip <= 1.0))) return KVQ_ERR_ARG;
    if (c->bucket < 0 || c->bucket % kT) return KVQ_ERR_SHAPE;
    if (c->bucket > 0 && !c->rope) return KVQ_ERR_ARG;
    if (!aligned(c->rope, 16)) return KVQ_ERR_ALIGN;
    if (!aligned(c->pages, 256) || !aligned(c->seq_len, 4) || !aligned(c->status, 4) || !aligned(c->v_rot, 16))
        return KVQ_ERR_ALIGN;
    return KVQ_OK;
}

int dtype_align(int dtype) { return dtype == KVQ_DTYPE_F32 ? 4 : 2; }

int cuda_status(cudaError_t e) { return e == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA; }

int num_sms() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    return n;
}

int check_decode_args(const kvq_cache *c, int Hq, int k) {
    int st = check_cache(c);
    if (st) return st;
    if (Hq < 1 || Hq % c->n_kv_heads) return KVQ_ERR_SHAPE;
    const int g = Hq / c->n_kv_heads;
    if (g != 1 && g != 2 && g != 4 && g != 8) return KVQ_ERR_SHAPE;
    if (k < 1 || k > kD) return KVQ_ERR_ARG;
    return KVQ_OK;
}

}  // namespace

extern "C" {

int kvq_version(void) { return 102; }

const char *kvq_status_string(int s) {
    switch (s) {
        case KVQ_OK: return "ok";
        case KVQ_ERR_ARG: return "invalid argument";
        case KVQ_ERR_SHAPE: return "unsupported shape";
        case KVQ_ERR_CAPACITY: return "capacity exceeded";
        case KVQ_ERR_WORKSPACE: return "workspace missing or too small";
        case KVQ_ERR_CUDA: return "CUDA error";
        case KVQ_ERR_ALIGN: return "misaligned pointer";
        default: return "unknown status";
    }
}

int kvq_num_buckets(const kvq_cache *c) {
    if (!c || c->capacity < 1 || c->bucket < 0 || (c->bucket > 0 && c->bucket % kT)) return 0;
    return buckets_of(*c);
}

size_t kvq_status_words(int batch, int n_kv_heads) {
    if (batch < 1 || n_kv_heads < 1) return 0;
    return 1 + (size_t)batch + (size_t)batch * n_kv_heads;
}

size_t kvq_page_bytes(int bits, int group) {
    if ((bits != 2 && bits != 4) || (group != kGroup && group != kD)) return 0;
    return (size_t)page_bytes(bits, kD / group);
}

size_t kvq_cache_bytes(const kvq_cache *c) {
    if (!c || c->batch < 1 || c->n_kv_heads < 1 || c->capacity < 1 || c->capacity % kT) return 0;
    if (c->head_dim != kD || (c->group != kGroup && c->group != kD) || (c->bits != 2 && c->bits != 4)) return 0;
    if (c->n_sink < 0 || c->n_recent < 0 || c->n_sink + c->n_recent > KVQ_MAX_PROTECTED) return 0;
    return (size_t)c->batch * c->n_kv_heads *
           ((size_t)(c->capacity / kT) * kvq_page_bytes(c->bits, c->group) +
            (size_t)(c->n_sink + c->n_recent) * kSlotBytes);
}

int kvq_cache_init(const kvq_cache *c, kvq_stream_t stream) {
    int st = check_cache(c);
    if (st) return st;
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e = cudaMemsetAsync(c->pages, 0, kvq_cache_bytes(c), s);
    if (e == cudaSuccess) e = cudaMemsetAsync(c->seq_len, 0, sizeof(int32_t) * c->batch, s);
    if (e == cudaSuccess)
        e = cudaMemsetAsync(c->status, 0, sizeof(uint32_t) * kvq_status_words(c->batch, c->n_kv_heads), s);
    return cuda_status(e);
}

int kvq_append(const kvq_cache *c, const void *K, const void *V, int dtype, int n_new,
               const double *A, kvq_stream_t stream) {
    int st = check_cache(c);
    if (st) return st;
    if (!K || !V || !A || n_new < 0) return KVQ_ERR_ARG;
    if (dtype != KVQ_DTYPE_F32 && dtype != KVQ_DTYPE_BF16) return KVQ_ERR_ARG;
    if (!aligned(K, dtype_align(dtype)) || !aligned(V, dtype_align(dtype)) || !aligned(A, 16))
        return KVQ_ERR_ALIGN;
    if (n_new > c->capacity) return KVQ_ERR_CAPACITY;
    if (n_new == 0) return KVQ_OK;
    return cuda_status(launch_append(*c, K, V, dtype, n_new, A, (cudaStream_t)stream));
}

int kvq_num_selected(float sparsity, int head_dim) {
    if (!(sparsity >= 0.f && sparsity < 1.f) || head_dim < 1) return -1;
    int k = (int)ceil((1.0 - (double)sparsity) * head_dim - 1e-9);
    if (k < 1) k = 1;
    return k > head_dim ? head_dim : k;
}

int kvq_select_channels(const kvq_cache *c, const void *q, int dtype, int n_q_heads,
                        const double *Ainvt, const double *delta, float sparsity, int32_t *idx,
                        float *qsel, float *qgsum, int *k_out, kvq_stream_t stream) {
    int st = check_cache(c);
    if (st) return st;
    if (!q || !Ainvt || !idx || !qsel || !qgsum) return KVQ_ERR_ARG;
    if (dtype != KVQ_DTYPE_F32 && dtype != KVQ_DTYPE_BF16) return KVQ_ERR_ARG;
    const int k = kvq_num_selected(sparsity, kD);
    if (k < 0) return KVQ_ERR_ARG;
    if (n_q_heads < 1 || n_q_heads % c->n_kv_heads || n_q_heads / c->n_kv_heads > 32) return KVQ_ERR_SHAPE;
    if (!aligned(q, dtype_align(dtype)) || !aligned(Ainvt, 16) || !aligned(delta, 8) || !aligned(idx, 4) ||
        !aligned(qsel, 4) || !aligned(qgsum, 4))
        return KVQ_ERR_ALIGN;
    if (k_out) *k_out = k;
    return cuda_status(
        launch_select(*c, q, dtype, n_q_heads, Ainvt, delta, k, idx, qsel, qgsum, (cudaStream_t)stream));
}

size_t kvq_decode_workspace(const kvq_cache *c, int n_q_heads, int k) {
    if (check_decode_args(c, n_q_heads, k)) return 0;
    const int S = decode_splits(*c, n_q_heads, k, num_sms());
    return decode_ws_bytes(*c, n_q_heads, S, true);
}

int kvq_decode_attn(const kvq_cache *c, int n_q_heads, const int32_t *idx, const float *qsel,
                    const float *qgsum, int k, float *out, void *ws, size_t ws_bytes,
                    kvq_stream_t stream) {
    int st = check_decode_args(c, n_q_heads, k);
    if (st) return st;
    if (!idx || !qsel || !qgsum || !out) return KVQ_ERR_ARG;
    if (!aligned(idx, 4) || !aligned(qsel, 4) || !aligned(qgsum, 4) || !aligned(out, 4)) return KVQ_ERR_ALIGN;
    const int sms = num_sms();
    if (sms <= 0) return KVQ_ERR_CUDA;
    const int S = decode_splits(*c, n_q_heads, k, sms);
    if (!ws || ws_bytes < decode_ws_bytes(*c, n_q_heads, S)) return KVQ_ERR_WORKSPACE;
    if (!aligned(ws, 16)) return KVQ_ERR_ALIGN;
    return cuda_status(launch_decode(*c, n_q_heads, idx, qsel, qgsum, k, out, ws, S, (cudaStream_t)stream));
}

int kvq_decode_attn_wait_bound(const kvq_cache *c, int n_q_heads, const int32_t *idx, const float *qsel,
                               const float *qgsum, int k, float *out, void *ws, size_t ws_bytes,
                               uint32_t wait_polls, kvq_stream_t stream) {
    int st = check_decode_args(c, n_q_heads, k);
    if (st) return st;
    if (!decode_uses_mma(*c, n_q_heads)) return KVQ_ERR_SHAPE;
    if (!idx || !qsel || !qgsum || !out) return KVQ_ERR_ARG;
    if (!aligned(idx, 4) || !aligned(qsel, 4) || !aligned(qgsum, 4) || !aligned(out, 4)) return KVQ_ERR_ALIGN;
    const int sms = num_sms();
    if (sms <= 0) return KVQ_ERR_CUDA;
    const int S = decode_splits(*c, n_q_heads, k, sms);
    if (!ws || ws_bytes < decode_ws_bytes(*c, n_q_heads, S)) return KVQ_ERR_WORKSPACE;
    if (!aligned(ws, 16)) return KVQ_ERR_ALIGN;
    return cuda_status(launch_decode(*c, n_q_heads, idx, qsel, qgsum, k, out, ws, S, (cudaStream_t)stream,
                                     (long long)wait_polls));
}

int kvq_decode_step(const kvq_cache *c, const void *q, const void *k_new, const void *v_new, int dtype,
                    int n_q_heads, int n_new, const double *A, const double *Ainvt, const double *delta,
                    float sparsity, int32_t *idx, float *qsel, float *qgsum, float *out, void *ws,
                    size_t ws_bytes, kvq_stream_t stream) {
    int st = check_cache(c);
    if (st) return st;
    if (!q || !A || !Ainvt || !idx || !qsel || !qgsum || !out || n_new < 0) return KVQ_ERR_ARG;
    if (n_new > 0 && (!k_new || !v_new)) return KVQ_ERR_ARG;
    if (dtype != KVQ_DTYPE_F32 && dtype != KVQ_DTYPE_BF16) return KVQ_ERR_ARG;
    const int k = kvq_num_selected(sparsity, kD);
    if (k < 0) return KVQ_ERR_ARG;
    st = check_decode_args(c, n_q_heads, k);
    if (st) return st;
    const size_t al = dtype_align(dtype);
    if (!aligned(q, al) || (n_new > 0 && (!aligned(k_new, al) || !aligned(v_new, al))) || !aligned(A, 16) ||
        !aligned(Ainvt, 16) || !aligned(delta, 8) || !aligned(idx, 4) || !aligned(qsel, 4) ||
        !aligned(qgsum, 4) || !aligned(out, 4))
        return KVQ_ERR_ALIGN;
    if (n_new > c->capacity) return KVQ_ERR_CAPACITY;
    const int sms = num_sms();
    if (sms <= 0) return KVQ_ERR_CUDA;
    const int S = decode_splits(*c, n_q_heads, k, sms);
    if (!ws || ws_bytes < decode_ws_bytes(*c, n_q_heads, S, true)) return KVQ_ERR_WORKSPACE;
    if (!aligned(ws, 16)) return KVQ_ERR_ALIGN;
    return cuda_status(launch_decode_step(*c, n_q_heads, q, k_new, v_new, dtype, n_new, A, Ainvt, delta, k, idx,
                                          qsel, qgsum, out, ws, S, (cudaStream_t)stream));
}

size_t kvq_bf16_decode_workspace(int B, int Hq, int Hkv, int N) {
    if (B < 1 || Hkv < 1 || Hq < 1 || Hq % Hkv || N < 0) return 0;
    return bf16_ws_bytes(B, Hq, bf16_splits(B, Hkv, N, num_sms()));
}

int kvq_bf16_decode_attn(const void *q, const void *K, const void *V, int B, int Hq, int Hkv, int N,
                         float *out, void *ws, size_t ws_bytes, kvq_stream_t stream) {
    if (!q || !out || B < 1 || Hkv < 1 || Hq < 1 || N < 0) return KVQ_ERR_ARG;
    if (N > 0 && (!K || !V)) return KVQ_ERR_ARG;
    if (Hq % Hkv) return KVQ_ERR_SHAPE;
    const int g = Hq / Hkv;
    if (g != 1 && g != 2 && g != 4 && g != 8) return KVQ_ERR_SHAPE;
    if (!aligned(q, 2) || !aligned(K, 16) || !aligned(V, 16) || !aligned(out, 4)) return KVQ_ERR_ALIGN;
    const int sms = num_sms();
    if (sms <= 0) return KVQ_ERR_CUDA;
    const int S = bf16_splits(B, Hkv, N, sms);
    if (!ws || ws_bytes < bf16_ws_bytes(B, Hq, S)) return KVQ_ERR_WORKSPACE;
    if (!aligned(ws, 16)) return KVQ_ERR_ALIGN;
    return cuda_status(launch_bf16_decode(q, K, V, B, Hq, Hkv, N, out, ws, S, (cudaStream_t)stream));
}

int kvq_copy_async(void *dst, const void *src, size_t bytes, kvq_stream_t stream) {
    if (bytes == 0) return KVQ_OK;
    if (!dst || !src) return KVQ_ERR_ARG;
    return cuda_status(cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDefault, (cudaStream_t)stream));
}

int kvq_read_status(const kvq_cache *c, uint32_t *flags, kvq_stream_t stream) {
    if (!c || !c->status || !flags) return KVQ_ERR_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e = cudaMemcpyAsync(flags, c->status, sizeof(uint32_t), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    return cuda_status(e);
}

}  // extern "C"
