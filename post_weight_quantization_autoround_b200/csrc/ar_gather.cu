// Minibatch assembly for block-by-block tuning: copies the calibration samples
// a step draws into one contiguous buffer, so the tuning step reads its tokens
// (and their reference outputs) as one [tokens][features] matrix.
//
// [AR] §8 preset table: every iteration works on a batch of 8 (4 in "fast")
// of the 128 calibration samples; [AR] §3 "Algorithm Flow" step 3-6 iterate on
// such batches ([AR] = "Low-Bit Quantization in Practice with vLLM: Core
// Mechanisms and Architectural Optimizations of AutoRound").
#include "ar_internal.h"

namespace ar {
namespace {

struct SampleIdx {
  int32_t v[kMaxGatherSamples];
};

// blockIdx.y = output sample; 16-byte vectors, streamed (read once)
__global__ void __launch_bounds__(256) gather_samples_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                                             int64_t sample_vec, SampleIdx idx) {
  const uint4* s = src + static_cast<int64_t>(idx.v[blockIdx.y]) * sample_vec;
  uint4* d = dst + static_cast<int64_t>(blockIdx.y) * sample_vec;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < sample_vec;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    d[i] = __ldcs(s + i);
}

}  // namespace

cudaError_t launch_gather_samples(const void* src, int64_t sample_bytes, const int32_t* idx, int n, void* dst,
                                  cudaStream_t stream) {
  SampleIdx si{};
  for (int i = 0; i < n; ++i) si.v[i] = idx[i];
  const int64_t sample_vec = sample_bytes / 16;
  const int64_t want = (sample_vec + 255) / 256;
  const int64_t cap = (8LL * num_sms() + n - 1) / n;  // about eight blocks per SM in total
  const int gx = static_cast<int>(want < cap ? (want > 0 ? want : 1) : cap);
  LaunchScope scope(stream, "gather_samples_kernel");
  gather_samples_kernel<<<dim3(gx, n), 256, 0, stream>>>(static_cast<const uint4*>(src), static_cast<uint4*>(dst),
                                                         sample_vec, si);
  return cudaGetLastError();
}

}  // namespace ar
