// thinkv_evict.cu -- evict to budget, slots back onto the free stacks.
//
// "ThinKV: Thought-Adaptive KV Cache Compression for Efficient Reasoning
// Models", explainer, Methodologie: TBE evicts tokens of less important
// thoughts; "Implementation Systeme: Pensee Continue (CT)": an evicted slot is
// only marked in the block table's eviction mask and becomes reusable by the
// next token of its thought type -- nothing is moved or compacted.
//
// One CTA.  The call is validated first (sequence range, duplicates, budget
// sign; all-or-nothing), then one warp per sequence takes its victims from the
// class FIFO heads in `order`, 32 at a time: slot ids are read coalesced, the
// bits of victims sharing a table entry are merged with __match_any_sync, an
// entry that loses its last live token leaves the live-page list (in victim
// order, by swap-with-last), and the victims are pushed on their class's free
// stack in victim order.  Each sequence's state is touched by one warp only.
#include <stdint.h>

#include "thinkv_common.cuh"
#include "thinkv_internal.h"

namespace thinkv {

namespace {

constexpr int kEvictThreads = 1024;
constexpr int kEvictWarps = kEvictThreads / 32;

struct Order {
  uint8_t c[4];
};

__global__ void __launch_bounds__(kEvictThreads, 1)
    evict_kernel(CacheView C, int32_t n, const int32_t* __restrict__ seq,
                 const int32_t* __restrict__ budget, Order order) {
  extern __shared__ uint32_t seen[];  // max_seqs bits
  __shared__ int s_err;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int max_seqs = C.L.max_seqs, nb_max = C.L.max_blocks_per_seq;
  const int64_t cap = (int64_t)nb_max * kPage;
  if (tid == 0) s_err = (*C.status != 0) ? -1 : 0;
  for (int i = tid; i < (max_seqs + 31) / 32; i += kEvictThreads) seen[i] = 0;
  __syncthreads();
  if (s_err != 0) return;
  for (int i = tid; i < n; i += kEvictThreads) {
    int s = seq[i];
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

  for (int i = warp; i < n; i += kEvictWarps) {
    const int s = seq[i];
    int remaining = C.live_count[s] - budget[i];
    if (remaining <= 0) continue;
    uint64_t* table = C.block_table + (int64_t)s * nb_max;
    uint64_t* llist = C.live_list + (int64_t)s * nb_max;
    int32_t* lidx = C.live_index + (int64_t)s * nb_max;
    int nlive = C.num_live[s];
    int evicted = 0;
    for (int o = 0; o < 3 && remaining > 0; ++o) {
      const int c = order.c[o];
      const int head = C.fifo_head[s * 3 + c];
      const int avail = C.fifo_tail[s * 3 + c] - head;
      const int take = min(avail, remaining);
      if (take <= 0) continue;
      const int32_t* ring = C.fifo + ((int64_t)s * 3 + c) * cap;
      int32_t* stack = C.free_slots + ((int64_t)s * 3 + c) * cap;
      const int top = C.free_top[s * 3 + c];
      for (int v0 = 0; v0 < take; v0 += 32) {
        const int v = v0 + lane;
        const bool valid = v < take;
        int32_t ts = valid ? ring[((int64_t)head + v) % cap] : 0;
        const int e = ts >> 4, slot = ts & 15;
        // merge the bits of victims that share an entry; the highest such lane
        // is the last victim of that entry in this batch
        const unsigned grp = __match_any_sync(0xFFFFFFFFu, valid ? e : -1 - lane);
        const uint32_t mybit = valid ? (1u << slot) : 0u;
        const uint32_t bits = __reduce_or_sync(grp, mybit);
        const bool last = valid && (31 - __clz(grp)) == lane;
        bool emptied = false;
        uint32_t page = 0;
        if (valid) {
          uint64_t ent = table[e];
          page = entry_page(ent);
          if (last) {
            uint32_t mask = entry_mask(ent) & ~bits;
            table[e] = (ent & 0x0000FFFFFFFFFFFFull) | ((uint64_t)mask << 48);
            emptied = (mask == 0);
          }
          C.slot_pos[c][(int64_t)page * kPage + slot] = -1;
          stack[top + v] = ts;
        }
        // entries emptied in this batch leave the live list in victim order
        unsigned ev = __ballot_sync(0xFFFFFFFFu, emptied);
        __syncwarp();
        while (ev) {
          const int src = __ffs(ev) - 1;
          const int ee = __shfl_sync(0xFFFFFFFFu, e, src);
          if (lane == 0) {
            const int at = lidx[ee];
            const int lastpos = --nlive;
            const uint64_t moved = llist[lastpos];
            llist[at] = moved;
            lidx[live_desc_entry(moved)] = at;
            lidx[ee] = -1;
          }
          nlive = __shfl_sync(0xFFFFFFFFu, nlive, 0);
          __syncwarp();
          ev &= ev - 1;
        }
      }
      if (lane == 0) {
        C.fifo_head[s * 3 + c] = head + take;
        C.free_top[s * 3 + c] = top + take;
      }
      remaining -= take;
      evicted += take;
    }
    if (lane == 0) {
      C.live_count[s] -= evicted;
      C.num_live[s] = nlive;
    }
    __syncwarp();
  }
}

}  // namespace

cudaError_t launch_evict(const CacheView& C, int32_t n, const int32_t* seq, const int32_t* budget,
                         const uint8_t order[3], cudaStream_t stream) {
  Order o;
  o.c[0] = order[0];
  o.c[1] = order[1];
  o.c[2] = order[2];
  o.c[3] = 0;
  const size_t seen_bytes = (size_t)((C.L.max_seqs + 31) / 32) * 4;
  evict_kernel<<<1, kEvictThreads, seen_bytes, stream>>>(C, n, seq, budget, o);
  return cudaGetLastError();
}

}  // namespace thinkv
