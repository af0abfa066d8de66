// thinkv_classify.cu -- thought tags from attention sparsity (mechanism only).
//
// "ThinKV: Thought-Adaptive KV Cache Compression for Efficient Reasoning
// Models", explainer, Methodologie, "Decomposition de la Pensee via la
// Parcimonie de l'Attention": a chain of thought splits into Reasoning,
// Execution and Transition thoughts by how sparse their attention is --
// Transition the sparsest, then Reasoning, Execution the least sparse.
//
// The sparsity of one decode step of a sequence is the mean over its query
// heads of the top-k attention mass that decode attention reports (a head
// whose probability sits on a few tokens has a mass near 1).  The tag is an
// integer decided by floating point, so the mean is one fp32 sum in head order
// divided by the head count, both rounded to nearest -- the same operations in
// the same order on any implementation.  One thread per sequence; the call is
// tiny next to decode (n * Hq * 4 bytes read).  The two thresholds are the
// calibration the pages leave to a real model.
#include <math.h>
#include <stdint.h>

#include "thinkv_common.cuh"
#include "thinkv_internal.h"

namespace thinkv {

namespace {

__global__ void classify_kernel(int32_t n, int32_t hq, const float* __restrict__ mass,
                                float theta_t, float theta_r, uint8_t* __restrict__ tags) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const float* m = mass + i * hq;
  float sum = 0.f;
  for (int h = 0; h < hq; ++h) sum = __fadd_rn(sum, m[h]);
  const float score = __fdiv_rn(sum, (float)hq);
  tags[i] = score >= theta_t ? THINKV_T : (score >= theta_r ? THINKV_R : THINKV_E);
}

}  // namespace

cudaError_t launch_classify(int32_t n, int32_t hq, const float* mass, float theta_t, float theta_r,
                            uint8_t* tags, cudaStream_t stream) {
  const int threads = 128;
  const int64_t blocks = ((int64_t)n + threads - 1) / threads;
  classify_kernel<<<(unsigned)blocks, threads, 0, stream>>>(n, hq, mass, theta_t, theta_r, tags);
  return cudaGetLastError();
}

}  // namespace thinkv
