// thinkv_victims.cu -- explicit victims: the eviction step a policy drives.
//
// "ThinKV: Thought-Adaptive KV Cache Compression for Efficient Reasoning
// Models", explainer, Methodologie, "Eviction Adaptative a la Pensee (TBE)"
// (segment-level eviction chosen by a policy) and "Implementation Systeme:
// Pensee Continue (CT)" (an evicted slot is marked in the block table and
// refilled in place by a later token of its type).  A policy that runs
// elsewhere names its victims; this call evicts them as TBE does its own.
//
// Victim i is the token at FIFO counter idx[i] of the class cls[i] FIFO of
// sequence seq[i] (head <= idx < tail).  Victims go in call order: mask bit
// cleared, start index -1, slot pushed onto its class's free stack, FIFO entry
// made a tombstone (-1), which the budget evict steps over.  A victim whose
// entry is already a tombstone (evicted before, or named earlier in the call)
// is skipped.  One CTA validates the call (all-or-nothing); then one warp per
// run of a sequence's victims takes them 32 at a time: repeats inside a batch
// by match on (class, counter), mask updates merged per table entry,
// free-stack ranks in victim order per class, emptied pages off the live list.
#include <stdint.h>

#include "thinkv_common.cuh"
#include "thinkv_internal.h"

namespace thinkv {

namespace {

constexpr int kVicThreads = 1024;
constexpr int kVicWarps = kVicThreads / 32;

__device__ inline unsigned lanes_below() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Block-wide exclusive scan of one int per thread (kVicThreads threads).
__device__ int vic_scan(int v, int* sh, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xFFFFFFFFu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sh[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = lane < kVicWarps ? sh[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xFFFFFFFFu, w, o);
      if (lane >= o) w += y;
    }
    sh[lane] = w;
  }
  __syncthreads();
  const int excl = (warp == 0 ? 0 : sh[warp - 1]) + x - v;
  *total = sh[kVicWarps - 1];
  __syncthreads();
  return excl;
}

__global__ void __launch_bounds__(kVicThreads, 1)
    evict_slots_kernel(CacheView C, int32_t n, const int32_t* __restrict__ seq,
                       const uint8_t* __restrict__ cls, const int32_t* __restrict__ idx,
                       int32_t* run_start) {
  extern __shared__ uint32_t seen[];  // max_seqs bits
  __shared__ int s_err;
  __shared__ int sh[40];
  __shared__ int s_nruns;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int max_seqs = C.L.max_seqs, nb_max = C.L.max_blocks_per_seq;
  const int64_t cap = (int64_t)nb_max * kPage;
  if (tid == 0) s_err = (*C.status != 0) ? -1 : 0;
  for (int i = tid; i < (max_seqs + 31) / 32; i += kVicThreads) seen[i] = 0;
  __syncthreads();
  if (s_err != 0) return;

  // ---- validate every victim; a sequence's victims must be one run ----
  int nruns = 0;
  for (int base = 0; base < n; base += kVicThreads) {
    const int i = base + tid;
    int start = 0;
    if (i < n) {
      const int s = seq[i], c = cls[i];
      bool bad = s < 0 || s >= max_seqs || c > 2;
      if (!bad) {
        const int k = idx[i];
        bad = k < C.fifo_head[s * 3 + c] || k >= C.fifo_tail[s * 3 + c];
      }
      start = (i == 0) || seq[i - 1] != s;
      if (!bad && start) {
        const uint32_t old = atomicOr(&seen[s >> 5], 1u << (s & 31));
        if (old & (1u << (s & 31))) bad = true;          // a sequence in two runs
      }
      if (bad) s_err = THINKV_ERR_INVALID;
    }
    int total;
    const int excl = vic_scan(start, sh, &total);
    if (start) run_start[nruns + excl] = i;
    nruns += total;
  }
  if (tid == 0) s_nruns = nruns;
  __syncthreads();
  if (s_err != 0) {
    if (tid == 0) set_status(C.status, s_err);
    return;
  }

  // ---- one warp per run ----
  const int R = s_nruns;
  for (int r = warp; r < R; r += kVicWarps) {
    const int start = run_start[r], end = r + 1 < R ? run_start[r + 1] : n;
    const int s = seq[start];
    uint64_t* table = C.block_table + (int64_t)s * nb_max;
    uint64_t* llist = C.live_list + (int64_t)s * nb_max;
    int32_t* lidx = C.live_index + (int64_t)s * nb_max;
    int top[3];
#pragma unroll
    for (int c = 0; c < 3; ++c) top[c] = C.free_top[s * 3 + c];
    int live = C.live_count[s], nlive = C.num_live[s];
    for (int b0 = start; b0 < end; b0 += 32) {
      const int i = b0 + lane;
      const bool in = i < end;
      const int c = in ? (int)cls[i] : 0;
      const int k = in ? idx[i] : 0;
      int32_t* ring = C.fifo + ((int64_t)s * 3 + c) * cap;
      const int32_t ts = in ? __ldcg(&ring[k % cap]) : -1;
      // a victim named twice in this batch acts once, from its first lane;
      // one named in an earlier batch finds its tombstone
      const unsigned same = __match_any_sync(
          0xFFFFFFFFu, in ? (long long)(((unsigned long long)(unsigned)c << 32) | (unsigned)k)
                          : (long long)(-1 - lane));
      const bool valid = in && ts >= 0 && (__ffs(same) - 1) == lane;
      const int ent = valid ? (ts >> 4) : -1, slot = ts & 15;
      // mask bits cleared per table entry by the entry's last victim lane
      const unsigned grp = __match_any_sync(0xFFFFFFFFu, valid ? ent : -1 - lane);
      const uint32_t bits = __reduce_or_sync(grp, valid ? (1u << slot) : 0u);
      const bool last = valid && (31 - __clz(grp)) == lane;
      // free-stack ranks in victim order, per class
      int crank = 0;
#pragma unroll
      for (int cc = 0; cc < 3; ++cc) {
        const unsigned cb = __ballot_sync(0xFFFFFFFFu, valid && c == cc);
        if (valid && c == cc) crank = top[cc] + __popc(cb & lanes_below());
        top[cc] += __popc(cb);
      }
      bool emptied = false;
      if (valid) {
        const uint64_t en = __ldcg(&table[ent]);
        const uint32_t page = entry_page(en);
        if (last) {
          const uint32_t mask = entry_mask(en) & ~bits;
          table[ent] = (en & 0x0000FFFFFFFFFFFFull) | ((uint64_t)mask << 48);
          emptied = (mask == 0);
        }
        if (page < (uint32_t)C.L.pool_pages[c]) C.slot_pos[c][(int64_t)page * kPage + slot] = -1;
        C.free_slots[((int64_t)s * 3 + c) * cap + (crank < cap ? crank : cap - 1)] = ts;
        ring[k % cap] = -1;                                // tombstone
      }
      live -= __popc(__ballot_sync(0xFFFFFFFFu, valid));
      unsigned ev = __ballot_sync(0xFFFFFFFFu, emptied);
      __syncwarp();
      while (ev) {                                        // emptied pages leave the live list
        const int src = __ffs(ev) - 1;
        const int ee = __shfl_sync(0xFFFFFFFFu, ent, src);
        if (lane == 0) {
          const int lastpos = nlive - 1;
          const int at = __ldcg(&lidx[ee]);
          const uint64_t moved = __ldcg(&llist[lastpos]);
          llist[at] = moved;
          lidx[live_desc_entry(moved)] = at;
          lidx[ee] = -1;
        }
        --nlive;
        __syncwarp();
        ev &= ev - 1;
      }
      __syncwarp();                                       // tombstones seen by the next batch
    }
    if (lane < 3) C.free_top[s * 3 + lane] = lane == 0 ? top[0] : (lane == 1 ? top[1] : top[2]);
    if (lane == 0) {
      C.live_count[s] = live;
      C.num_live[s] = nlive;
    }
  }
}

}  // namespace

cudaError_t launch_evict_slots(const CacheView& C, int32_t n, const int32_t* seq, const uint8_t* cls,
                               const int32_t* idx, int32_t* run_start, cudaStream_t stream) {
  const size_t seen_bytes = (size_t)((C.L.max_seqs + 31) / 32) * 4;
  if (seen_bytes > 48 * 1024) {
    const cudaError_t e = cudaFuncSetAttribute(evict_slots_kernel,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)seen_bytes);
    if (e != cudaSuccess) return e;
  }
  evict_slots_kernel<<<1, kVicThreads, seen_bytes, stream>>>(C, n, seq, cls, idx, run_start);
  return cudaGetLastError();
}

}  // namespace thinkv
