// thinkv_evict_seq.cuh -- the budget eviction of one sequence by one warp,
// shared by the evict kernels and the one-launch append + evict.
//
// "ThinKV: Thought-Adaptive KV Cache Compression for Efficient Reasoning
// Models", explainer, Methodologie: TBE evicts tokens of less important
// thoughts; "Implementation Systeme: Pensee Continue (CT)": an evicted slot is
// only marked in the block table's eviction mask and becomes reusable by the
// next token of its thought type.
#ifndef THINKV_EVICT_SEQ_CUH
#define THINKV_EVICT_SEQ_CUH

#include <stdint.h>

#include "thinkv_common.cuh"
#include "thinkv_internal.h"

namespace thinkv {
namespace {

// Evicts sequence s down to `bud` live tokens (one warp).  The class order is
// packed one class per byte.  All of s's counters are loaded at once (with
// the sticky status when check_status: a set status makes this a no-op).
// Victims are the oldest live entries of the first class in order that has
// one, then the next class: each class FIFO is scanned from its head 32
// entries at a time; -1 entries are tombstones (tokens TBE evicted away from
// the head), stepped over and consumed like the victims before them.
__device__ inline void evict_seq(const CacheView& C, int s, int bud, uint32_t order,
                                 bool check_status) {
  const int lane = threadIdx.x & 31;
  const int nb_max = C.L.max_blocks_per_seq;
  const int64_t cap = (int64_t)nb_max * kPage;
  // lanes 0-2: FIFO heads, 3-5: FIFO tails, 6-8: stack tops (classes in
  // order), 9: live_count, 10: num_live
  int val = 0;
  {
    const int o = lane % 3, c = (int)((order >> (8 * o)) & 0xFFu);
    if (lane < 3) val = C.fifo_head[s * 3 + c];
    else if (lane < 6) val = C.fifo_tail[s * 3 + c];
    else if (lane < 9) val = C.free_top[s * 3 + c];
    else if (lane == 9) val = C.live_count[s];
    else if (lane == 10) val = C.num_live[s];
    else if (lane == 11 && check_status) val = *C.status;
  }
  if (check_status && __shfl_sync(0xFFFFFFFFu, val, 11) != 0) return;
  const int live = __shfl_sync(0xFFFFFFFFu, val, 9);
  int nlive = __shfl_sync(0xFFFFFFFFu, val, 10);
  int remaining = live - bud;
  if (remaining <= 0) return;
  uint64_t* table = C.block_table + (int64_t)s * nb_max;
  uint64_t* llist = C.live_list + (int64_t)s * nb_max;
  int32_t* lidx = C.live_index + (int64_t)s * nb_max;
  int total = 0;
  int new_head = 0, new_top = 0;                     // lane o < 3 keeps class o's values
  for (int o = 0; o < 3; ++o) {
    const int c = (int)((order >> (8 * o)) & 0xFFu);
    int idx = __shfl_sync(0xFFFFFFFFu, val, o);
    const int tail = __shfl_sync(0xFFFFFFFFu, val, 3 + o);
    int top = __shfl_sync(0xFFFFFFFFu, val, 6 + o);
    const int32_t* ring = C.fifo + ((int64_t)s * 3 + c) * cap;
    int32_t* stack = C.free_slots + ((int64_t)s * 3 + c) * cap;
    while (remaining > 0 && idx < tail) {
      const int cnt = min(32, tail - idx);
      const int32_t ts = lane < cnt ? ring[((int64_t)idx + lane) % cap] : -1;
      const unsigned lbal = __ballot_sync(0xFFFFFFFFu, ts >= 0);
      const int rank = __popc(lbal & ((1u << lane) - 1u));
      const bool valid = ts >= 0 && rank < remaining;
      const unsigned vbal = __ballot_sync(0xFFFFFFFFu, valid);
      const int nv = __popc(vbal);
      // the quota reached: consumed up to the last victim; else the whole chunk
      const int consumed = (nv == remaining) ? 32 - __clz(vbal) : cnt;
      const int e = valid ? (ts >> 4) : -1, slot = ts & 15;
      // merge the bits of victims that share an entry (entries are class-pure);
      // the highest such lane writes the entry
      const unsigned grp = __match_any_sync(0xFFFFFFFFu, valid ? e : -1 - lane);
      const uint32_t bits = __reduce_or_sync(grp, valid ? (1u << slot) : 0u);
      const bool last = valid && (31 - __clz(grp)) == lane;
      bool emptied = false;
      if (valid) {
        // through L2: an earlier batch may have rewritten this entry
        const uint64_t ent = __ldcg(&table[e]);
        const uint32_t page = entry_page(ent);
        if (last) {
          const uint32_t mask = entry_mask(ent) & ~bits;
          table[e] = (ent & 0x0000FFFFFFFFFFFFull) | ((uint64_t)mask << 48);
          emptied = (mask == 0);
        }
        C.slot_pos[c][(int64_t)page * kPage + slot] = -1;
        stack[top + rank] = ts;
      }
      // entries emptied in this batch leave the live list in victim order
      unsigned ev = __ballot_sync(0xFFFFFFFFu, emptied);
      __syncwarp();
      while (ev) {
        const int src = __ffs(ev) - 1;
        const int ee = __shfl_sync(0xFFFFFFFFu, e, src);
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
      top += nv;
      remaining -= nv;
      total += nv;
      idx += consumed;
    }
    if (lane == o) {
      new_head = idx;
      new_top = top;
    }
  }
  if (lane < 3) {
    const int c = (int)((order >> (8 * lane)) & 0xFFu);
    C.fifo_head[s * 3 + c] = new_head;
    C.free_top[s * 3 + c] = new_top;
  }
  if (lane == 0) {
    C.live_count[s] = live - total;
    C.num_live[s] = nlive;
  }
}

}  // namespace
}  // namespace thinkv

#endif
