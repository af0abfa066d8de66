// thinkv_evict.cu -- evict to budget, slots back onto the free stacks.
//
// "ThinKV: Thought-Adaptive KV Cache Compression for Efficient Reasoning
// Models", explainer, Methodologie: TBE evicts tokens of less important
// thoughts; "Implementation Systeme: Pensee Continue (CT)": an evicted slot is
// only marked in the block table's eviction mask and becomes reusable by the
// next token of its thought type -- nothing is moved or compacted.
//
// The call is validated first (sequence range, duplicates, budget sign;
// all-or-nothing), then one warp per sequence takes its victims from the
// class FIFO heads in `order`, 32 at a time: slot ids are read coalesced,
// tombstones left by TBE are stepped over, the bits of victims sharing a table
// entry are merged with __match_any_sync, an entry that loses its last live
// token leaves the live-page list (in victim order, by swap-with-last), and
// the victims are pushed on their class's free stack in victim order.  Each
// sequence's state is touched by one warp only.
#include <stdint.h>

#include "thinkv_common.cuh"
#include "thinkv_evict_seq.cuh"
#include "thinkv_internal.h"

namespace thinkv {

namespace {

constexpr int kEvictThreads = 1024;
constexpr int kEvictWarps = kEvictThreads / 32;


// Calls of any size: one CTA validates the call (all-or-nothing), then a warp
// per sequence evicts it (evict_seq).  With `runs`, seq and budget are an
// append's token arrays: only the first token of each run of a sequence names
// it (and its budget).
__global__ void __launch_bounds__(kEvictThreads, 1)
    evict_kernel(CacheView C, int32_t n, const int32_t* __restrict__ seq,
                 const int32_t* __restrict__ budget, uint32_t order, bool runs) {
  extern __shared__ uint32_t seen[];  // max_seqs bits
  __shared__ int s_err;
  const int tid = threadIdx.x, warp = tid >> 5;
  const int max_seqs = C.L.max_seqs;
  if (tid == 0) s_err = (*C.status != 0) ? -1 : 0;
  for (int i = tid; i < (max_seqs + 31) / 32; i += kEvictThreads) seen[i] = 0;
  __syncthreads();
  if (s_err != 0) return;
  for (int i = tid; i < n; i += kEvictThreads) {
    int s = seq[i];
    if (runs && i > 0 && seq[i - 1] == s) continue;
    bool bad = s < 0 || s >= max_seqs || budget[i] < 0;
    if (!bad) {
      uint32_t old = atomicOr(&seen[s >> 5], 1u << (s & 31));
      if (old & (1u << (s & 31))) bad = true;
    }
    if (bad) s_err = THINKV_ERR_INVALID;
  }
  __syncthreads();
  if (s_err != 0) {
    if (tid == 0) set_status(C.status, s_err);
    return;
  }
  for (int i = warp; i < n; i += kEvictWarps)
    if (!runs || i == 0 || seq[i - 1] != seq[i]) evict_seq(C, seq[i], budget[i], order, false);
}


// ---------------------------------------------------------------------------
// small calls (n <= kSmallEvict sequences, e.g. a decode step): one warp per
// sequence over many CTAs.  Every CTA validates the whole call itself (the
// same verdict everywhere, so the call stays all-or-nothing without a
// grid-wide barrier); sequences share no state, so the warps are independent.
// ---------------------------------------------------------------------------
constexpr int kSmallEvict = 512;
constexpr int kSmallEvictThreads = 256;
constexpr int kSmallEvictWarps = kSmallEvictThreads / 32;


__global__ void __launch_bounds__(kSmallEvictThreads)
    evict_small_kernel(CacheView C, int32_t n, const int32_t* __restrict__ seq,
                       const int32_t* __restrict__ budget, uint32_t order) {
  extern __shared__ uint32_t seen[];  // max_seqs bits
  __shared__ int s_err;
  __shared__ int my_seq[kSmallEvictWarps], my_bud[kSmallEvictWarps];
  const int tid = threadIdx.x, warp = tid >> 5;
  const int max_seqs = C.L.max_seqs;
  const int first = blockIdx.x * kSmallEvictWarps;
  pdl_launch_dependents();
  // ---- the call's own inputs (before the previous kernel has finished) ----
  for (int i = tid; i < (max_seqs + 31) / 32; i += kSmallEvictThreads) seen[i] = 0;
  if (tid == 0) s_err = 0;
  __syncthreads();
  for (int i = tid; i < n; i += kSmallEvictThreads) {
    const int s = seq[i], b = budget[i];
    bool bad = s < 0 || s >= max_seqs || b < 0;
    if (!bad) {
      const uint32_t old = atomicOr(&seen[s >> 5], 1u << (s & 31));
      if (old & (1u << (s & 31))) bad = true;
    }
    if (bad) s_err = THINKV_ERR_INVALID;
    if (i >= first && i < first + kSmallEvictWarps) {
      my_seq[i - first] = s;
      my_bud[i - first] = b;
    }
  }
  __syncthreads();
  // ---- cache state: only once the previous kernel is done ----
  pdl_wait();
  if (s_err != 0) {
    if (blockIdx.x == 0 && tid == 0) set_status(C.status, s_err);
    return;
  }
  const int i = first + warp;
  if (i < n) evict_seq(C, my_seq[warp], my_bud[warp], order, true);
}
}  // namespace

cudaError_t launch_evict(const CacheView& C, int32_t n, const int32_t* seq, const int32_t* budget,
                         const uint8_t order[3], cudaStream_t stream) {
  const uint32_t packed = (uint32_t)order[0] | ((uint32_t)order[1] << 8) | ((uint32_t)order[2] << 16);
  const size_t seen_bytes = (size_t)((C.L.max_seqs + 31) / 32) * 4;
  if (n <= kSmallEvict) {
    const int grid = (n + kSmallEvictWarps - 1) / kSmallEvictWarps;
    return launch_pdl(evict_small_kernel, dim3(grid), dim3(kSmallEvictThreads), seen_bytes, stream,
                      C, n, seq, budget, packed);
  }
  evict_kernel<<<1, kEvictThreads, seen_bytes, stream>>>(C, n, seq, budget, packed, false);
  return cudaGetLastError();
}

cudaError_t launch_evict_runs(const CacheView& C, int32_t n, const int32_t* seq, const int32_t* budget,
                              const uint8_t order[3], cudaStream_t stream) {
  const uint32_t packed = (uint32_t)order[0] | ((uint32_t)order[1] << 8) | ((uint32_t)order[2] << 16);
  const size_t seen_bytes = (size_t)((C.L.max_seqs + 31) / 32) * 4;
  evict_kernel<<<1, kEvictThreads, seen_bytes, stream>>>(C, n, seq, budget, packed, true);
  return cudaGetLastError();
}

}  // namespace thinkv
