// Internal definitions shared by the kvq CUDA kernels (sm_100a).
// Page layout and arithmetic conventions are documented in include/kvq.h.
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "kvq.h"

namespace kvq {

constexpr int kD = 128;        // head dimension
constexpr int kT = 128;        // tokens per page
constexpr int kGroup = 32;     // channels per quantization group
constexpr int kNG = kD / kGroup;

__host__ __device__ constexpr int row_bytes(int bits) { return kT * bits / 8; }
__host__ __device__ constexpr int off_vcodes(int bits) { return 128 * row_bytes(bits); }
__host__ __device__ constexpr int off_ch0(int bits) { return 256 * row_bytes(bits); }
__host__ __device__ constexpr int off_kmeta(int bits) { return off_ch0(bits) + 256; }
__host__ __device__ constexpr int off_vmeta(int bits) { return off_kmeta(bits) + 2048; }
__host__ __device__ constexpr int page_bytes(int bits) { return off_vmeta(bits) + 2048; }
// bytes from the value codes to the end of the page: what every decode step
// reads in full (value codes, channel 0, key and value metadata)
__host__ __device__ constexpr int fixed_bytes(int bits) { return page_bytes(bits) - off_vcodes(bits); }

// log2(e) / sqrt(128): scores are kept in the base-2 exponent domain
constexpr float kScoreScaleLog2 = 0.12751743074460787f;

// ------------------------------------------------------------ conversions
__device__ __forceinline__ double in_to_double(float x) { return (double)x; }
__device__ __forceinline__ double in_to_double(uint16_t bf) {
    return (double)__uint_as_float(((uint32_t)bf) << 16);
}
__device__ __forceinline__ float in_to_float(float x) { return x; }
__device__ __forceinline__ float in_to_float(uint16_t bf) {
    return __uint_as_float(((uint32_t)bf) << 16);
}

// ------------------------------------------------------------ cp.async
__device__ __forceinline__ void cp_async16(void *smem_dst, const void *gmem_src) {
    uint32_t d = (uint32_t)__cvta_generic_to_shared(smem_dst);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(d), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory"); }

// ------------------------------------------------------------ split plan
struct SplitPlan {
    int n_splits;
};

}  // namespace kvq

// launchers implemented in the .cu files (host side, called by kvq_api.cu)
namespace kvq {
cudaError_t launch_append(const kvq_cache &c, const void *K, const void *V, int dtype, int n_new,
                          const double *A, cudaStream_t st);
cudaError_t launch_select(const kvq_cache &c, const void *q, int dtype, int Hq, const double *Ainvt,
                          int k, int32_t *idx, float *qsel, float *qgsum, cudaStream_t st);
int decode_splits(const kvq_cache &c, int Hq, int k, int num_sms);
size_t decode_ws_bytes(const kvq_cache &c, int Hq, int n_splits);
cudaError_t launch_decode(const kvq_cache &c, int Hq, const int32_t *idx, const float *qsel,
                          const float *qgsum, int k, float *out, void *ws, int n_splits,
                          cudaStream_t st);
int bf16_splits(int B, int Hkv, int N, int num_sms);
size_t bf16_ws_bytes(int B, int Hq, int n_splits);
cudaError_t launch_bf16_decode(const void *q, const void *K, const void *V, int B, int Hq, int Hkv,
                               int N, float *out, void *ws, int n_splits, cudaStream_t st);
}  // namespace kvq
