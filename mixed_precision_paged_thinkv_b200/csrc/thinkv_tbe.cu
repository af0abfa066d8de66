// thinkv_tbe.cu -- TBE: segment-level eviction on Transition thoughts.
//
// "ThinKV: Thought-Adaptive KV Cache Compression for Efficient Reasoning
// Models", explainer, Methodologie, "Eviction Adaptative a la Pensee (TBE)":
// when a Transition thought appears, tokens of the earlier, less critical
// Reasoning and Execution segments are evicted progressively along an
// annealing schedule (retention 64, then 32, then 16), a segment at a time;
// the explainer's "Astuce B" adds that a small safety net of Transition
// tokens is always kept.  Readings (the pages give no more):
//   - a segment is a maximal run of consecutive tokens of a sequence with one
//     tag, in append order; a T event is the first token of a new T segment;
//   - at a T event each earlier R or E segment takes the next schedule step
//     (its k-th event keeps at most schedule[min(k, 3) - 1] tokens) and the
//     earlier T segments keep only the t_min most recent live T tokens;
//   - a segment gives up its oldest live tokens first, so its live tokens
//     are always the newest ones; victims go in segment order, then token
//     order, onto their class's free stack (CT: the slot is refilled in place);
//   - a victim need not be at its FIFO head: its FIFO entry becomes a
//     tombstone (-1), which the budget evict steps over.
//
// The call follows an append and takes the same token arrays.  One CTA: it
// validates the call (all-or-nothing, including the segment table's room),
// then one warp per sequence run records the run's segments -- the FIFO
// counter of a segment's first token, lo, follows from the FIFO tail the
// append left -- and handles the run's T events in order.  A segment's live
// tokens are the FIFO entries [max(lo + trim, head), lo + len).  Segments that
// no event can change any more (R/E at the last schedule step within its
// retention, T with nothing live) are skipped by a per-sequence frontier.
#include <stdint.h>

#include "thinkv_common.cuh"
#include "thinkv_internal.h"

namespace thinkv {

namespace {

constexpr int kTbeThreads = 1024;
constexpr int kTbeWarps = kTbeThreads / 32;

struct TbeView {
  int4* seg;          // [max_seqs][cap]: (class | level << 8, lo, len, trim)
  int32_t* nseg;      // [max_seqs]
  int32_t* settled;   // [max_seqs] segments before it can no longer change
};

__device__ inline unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Block-wide exclusive scan of one int per thread (kTbeThreads threads).
__device__ int block_scan(int v, int* sh, int* total) {
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
    int w = lane < kTbeWarps ? sh[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xFFFFFFFFu, w, o);
      if (lane >= o) w += y;
    }
    sh[lane] = w;
  }
  __syncthreads();
  const int excl = (warp == 0 ? 0 : sh[warp - 1]) + x - v;
  *total = sh[kTbeWarps - 1];
  __syncthreads();
  return excl;
}

// Per-warp view of one sequence's eviction counters while TBE runs.
struct SeqCounters {
  int head[3], top[3];
  int live, nlive;
};

// The T event that opens segment e of sequence s (one warp).
__device__ void tbe_event(const CacheView& C, const TbeView& T, int s, int e, int t_min,
                          const int (&sched)[3], SeqCounters& K) {
  const int lane = threadIdx.x & 31;
  const int nb_max = C.L.max_blocks_per_seq;
  const int64_t cap = (int64_t)nb_max * kPage;
  int4* segs = T.seg + (int64_t)s * cap;
  uint64_t* table = C.block_table + (int64_t)s * nb_max;
  uint64_t* llist = C.live_list + (int64_t)s * nb_max;
  int32_t* lidx = C.live_index + (int64_t)s * nb_max;
  const int settled0 = T.settled[s];
  auto live_of = [&](const int4& g, int* first) {
    const int c = g.x & 0xFF;
    const int hd = c == 0 ? K.head[0] : (c == 1 ? K.head[1] : K.head[2]);
    const int a = g.y + g.w;
    *first = a > hd ? a : hd;
    const int l = g.y + g.z - *first;
    return l > 0 ? l : 0;
  };
  // live tokens of the earlier T segments (the safety net counts from the newest)
  int t_total = 0;
  for (int j0 = settled0; j0 < e; j0 += 32) {
    const int j = j0 + lane;
    int x = 0;
    if (j < e) {
      const int4 g = segs[j];
      int first;
      if ((g.x & 0xFF) == THINKV_T) x = live_of(g, &first);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xFFFFFFFFu, x, o);
    t_total += x;
  }
  int t_before = 0;            // live T tokens of the segments before this chunk
  int settled = settled0;
  bool settling = true;        // every segment so far is final
  for (int j0 = settled0; j0 < e; j0 += 32) {
    const int j = j0 + lane;
    const bool in = j < e;
    int4 g = in ? segs[j] : make_int4(0, 0, 0, 0);
    const int c = g.x & 0xFF;
    int level = (g.x >> 8) & 0xFF;
    int first = 0;
    const int live = in ? live_of(g, &first) : 0;
    const int tl = (in && c == THINKV_T) ? live : 0;
    int tin = tl;                                       // inclusive prefix of T live in the chunk
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xFFFFFFFFu, tin, o);
      if (lane >= o) tin += y;
    }
    int x = 0;                                          // victims of segment j
    if (in) {
      if (c == THINKV_T) {
        const int newer = t_total - (t_before + tin);   // live T tokens of later T segments
        int keep = t_min - newer;
        keep = keep < 0 ? 0 : (keep > live ? live : keep);
        x = live - keep;
      } else {
        level = level < 3 ? level + 1 : 3;
        const int keep = sched[level - 1];
        x = live > keep ? live - keep : 0;
        g.x = c | (level << 8);
      }
      if (x > 0) g.w = first + x - g.y;
      segs[j] = g;
    }
    t_before += __shfl_sync(0xFFFFFFFFu, tin, 31);
    // segments no later event can change: the frontier moves past them
    const bool fin = in && (c == THINKV_T ? live - x == 0 : (level == 3 && live - x <= sched[2]));
    if (settling) {
      const unsigned nf = __ballot_sync(0xFFFFFFFFu, in && !fin);
      const int cnt = min(32, e - j0);
      if (nf) {
        settled = j0 + __ffs(nf) - 1;
        settling = false;
      } else {
        settled = j0 + cnt;
      }
    }
    // the chunk's victims, flattened in segment then token order
    int pre = x;                                        // inclusive prefix of x
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xFFFFFFFFu, pre, o);
      if (lane >= o) pre += y;
    }
    const int X = __shfl_sync(0xFFFFFFFFu, pre, 31);
    for (int v0 = 0; v0 < X; v0 += 32) {
      const int v = v0 + lane;
      const bool valid = v < X;
      // the chunk lane (segment) that owns victim v: the first with pre > v
      int lo = 0, hi = 31;
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        const int pm = __shfl_sync(0xFFFFFFFFu, pre, mid);
        if (pm > v) hi = mid; else lo = mid + 1;
      }
      const int owner = lo;
      const int pre_o = __shfl_sync(0xFFFFFFFFu, pre, owner);
      const int x_o = __shfl_sync(0xFFFFFFFFu, x, owner);
      const int first_o = __shfl_sync(0xFFFFFFFFu, first, owner);
      const int c_o = __shfl_sync(0xFFFFFFFFu, c, owner);
      const int64_t fidx = (int64_t)first_o + (v - (pre_o - x_o));
      int32_t* ring = C.fifo + ((int64_t)s * 3 + c_o) * cap;
      const int32_t ts = valid ? ring[fidx % cap] : 0;
      const int ent = valid ? (ts >> 4) : -1, slot = ts & 15;
      const unsigned grp = __match_any_sync(0xFFFFFFFFu, valid ? ent : -1 - lane);
      const uint32_t bits = __reduce_or_sync(grp, valid ? (1u << slot) : 0u);
      const bool last = valid && (31 - __clz(grp)) == lane;
      bool emptied = false;
      int crank = 0;
#pragma unroll
      for (int cc = 0; cc < 3; ++cc) {
        const unsigned cb = __ballot_sync(0xFFFFFFFFu, valid && c_o == cc);
        if (c_o == cc) crank = (cc == 0 ? K.top[0] : (cc == 1 ? K.top[1] : K.top[2])) +
                               __popc(cb & lanemask_lt());
        if (cc == 0) K.top[0] += __popc(cb);
        else if (cc == 1) K.top[1] += __popc(cb);
        else K.top[2] += __popc(cb);
      }
      if (valid) {
        // ts >= 0 and its page in range hold whenever the calls follow the
        // documented order; the checks keep a misordered call in bounds
        const uint64_t en = ts >= 0 ? __ldcg(&table[ent]) : 0ull;
        const uint32_t page = entry_page(en);
        if (last && ts >= 0) {
          const uint32_t mask = entry_mask(en) & ~bits;
          table[ent] = (en & 0x0000FFFFFFFFFFFFull) | ((uint64_t)mask << 48);
          emptied = (mask == 0);
        }
        if (ts >= 0 && page < (uint32_t)C.L.pool_pages[c_o])
          C.slot_pos[c_o][(int64_t)page * kPage + slot] = -1;
        C.free_slots[((int64_t)s * 3 + c_o) * cap + (crank < cap ? crank : cap - 1)] = ts;
        ring[fidx % cap] = -1;                           // tombstone
      }
      unsigned ev = __ballot_sync(0xFFFFFFFFu, emptied);
      __syncwarp();
      while (ev) {
        const int src = __ffs(ev) - 1;
        const int ee = __shfl_sync(0xFFFFFFFFu, ent, src);
        if (lane == 0) {
          const int lastpos = K.nlive - 1;
          const int at = __ldcg(&lidx[ee]);
          const uint64_t moved = __ldcg(&llist[lastpos]);
          llist[at] = moved;
          lidx[live_desc_entry(moved)] = at;
          lidx[ee] = -1;
        }
        --K.nlive;
        __syncwarp();
        ev &= ev - 1;
      }
    }
    K.live -= X;
  }
  if (lane == 0) T.settled[s] = settled;
  __syncwarp();
}

__global__ void __launch_bounds__(kTbeThreads, 1)
    tbe_kernel(CacheView C, TbeView T, int32_t n, const int32_t* __restrict__ seq,
               const int32_t* __restrict__ pos, const uint8_t* __restrict__ tag, int32_t t_min,
               int4 schedule, int32_t* run_start) {
  extern __shared__ uint32_t seen[];  // max_seqs bits
  __shared__ int s_err;
  __shared__ int sh[40];
  __shared__ int s_nruns;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int max_seqs = C.L.max_seqs, nb_max = C.L.max_blocks_per_seq;
  const int64_t cap = (int64_t)nb_max * kPage;
  const int sched[3] = {schedule.x, schedule.y, schedule.z};
  if (tid == 0) s_err = (*C.status != 0) ? -1 : 0;
  for (int i = tid; i < (max_seqs + 31) / 32; i += kTbeThreads) seen[i] = 0;
  __syncthreads();
  if (s_err != 0) return;

  // ---- validate (the append's rules), mark run starts ----
  int nruns = 0;
  for (int base = 0; base < n; base += kTbeThreads) {
    const int i = base + tid;
    int start = 0;
    if (i < n) {
      const int s = seq[i], c = tag[i], p = pos[i];
      bool bad = s < 0 || s >= max_seqs || c > 2 || p < 0;
      start = (i == 0) || seq[i - 1] != s;
      if (!bad && !start && p <= pos[i - 1]) bad = true;
      if (!bad && start) {
        const uint32_t old = atomicOr(&seen[s >> 5], 1u << (s & 31));
        if (old & (1u << (s & 31))) bad = true;
      }
      if (bad) s_err = THINKV_ERR_INVALID;
    }
    int total;
    const int excl = block_scan(start, sh, &total);
    if (start) run_start[nruns + excl] = i;
    nruns += total;
  }
  if (tid == 0) s_nruns = nruns;
  __syncthreads();
  if (s_err != 0) {
    if (tid == 0) set_status(C.status, s_err);
    return;
  }
  const int R = s_nruns;
  // ---- room in every sequence's segment table; the run's tokens must be the
  //      newest of their class FIFOs (the append of this call put them there) ----
  for (int r = warp; r < R; r += kTbeWarps) {
    const int start = run_start[r], end = r + 1 < R ? run_start[r + 1] : n;
    const int s = seq[start];
    const int ns0 = T.nseg[s];
    const int last_cls = ns0 > 0 ? (T.seg[(int64_t)s * cap + ns0 - 1].x & 0xFF) : -1;
    int added = 0, cnt[3] = {0, 0, 0};
    for (int b0 = start; b0 < end; b0 += 32) {
      const int i = b0 + lane;
      const int c = i < end ? (int)tag[i] : -1;
      const bool st = i < end && c != (i == start ? last_cls : (int)tag[i - 1]);
      added += __popc(__ballot_sync(0xFFFFFFFFu, st));
#pragma unroll
      for (int cc = 0; cc < 3; ++cc) cnt[cc] += __popc(__ballot_sync(0xFFFFFFFFu, c == cc));
    }
    if (lane == 0) {
      bool bad = (int64_t)ns0 + added > cap;
#pragma unroll
      for (int cc = 0; cc < 3; ++cc)
        bad |= cnt[cc] > C.fifo_tail[s * 3 + cc] - C.fifo_head[s * 3 + cc];
      if (bad) s_err = THINKV_ERR_INVALID;
    }
  }
  __syncthreads();
  if (s_err != 0) {
    if (tid == 0) set_status(C.status, s_err);
    return;
  }

  // ---- per run: record its segments, then its T events in order ----
  for (int r = warp; r < R; r += kTbeWarps) {
    const int start = run_start[r], end = r + 1 < R ? run_start[r + 1] : n;
    const int s = seq[start];
    int4* segs = T.seg + (int64_t)s * cap;
    SeqCounters K;
    int tail[3];
#pragma unroll
    for (int c = 0; c < 3; ++c) {
      K.head[c] = C.fifo_head[s * 3 + c];
      K.top[c] = C.free_top[s * 3 + c];
      tail[c] = C.fifo_tail[s * 3 + c];
    }
    K.live = C.live_count[s];
    K.nlive = C.num_live[s];
    const int ns0 = T.nseg[s];
    const int last_cls = ns0 > 0 ? (segs[ns0 - 1].x & 0xFF) : -1;
    // the run's class counts: its class-c tokens took FIFO counters tail - cnt ..
    int cnt[3] = {0, 0, 0};
    for (int b0 = start; b0 < end; b0 += 32) {
      const int i = b0 + lane;
      const int c = i < end ? (int)tag[i] : -1;
#pragma unroll
      for (int cc = 0; cc < 3; ++cc) cnt[cc] += __popc(__ballot_sync(0xFFFFFFFFu, c == cc));
    }
    int next[3] = {tail[0] - cnt[0], tail[1] - cnt[1], tail[2] - cnt[2]};
    int nseg = ns0;
    for (int b0 = start; b0 < end; b0 += 32) {
      const int i = b0 + lane;
      const bool in = i < end;
      const int c = in ? (int)tag[i] : 0;
      int idx = 0;
      unsigned cb[3];
#pragma unroll
      for (int cc = 0; cc < 3; ++cc) {
        cb[cc] = __ballot_sync(0xFFFFFFFFu, in && c == cc);
        if (in && c == cc) idx = next[cc] + __popc(cb[cc] & lanemask_lt());
      }
#pragma unroll
      for (int cc = 0; cc < 3; ++cc) next[cc] += __popc(cb[cc]);
      const bool st = in && c != (i == start ? last_cls : (int)tag[i - 1]);
      const unsigned sb = __ballot_sync(0xFFFFFFFFu, st);
      // segment of each token: the last start at or before it (or the open one)
      const int sidx = nseg + __popc(sb & (lanemask_lt() | (1u << lane))) - 1;
      if (st) segs[sidx] = make_int4(c, idx, 0, 0);
      __syncwarp();
      // lengths: the tokens of each segment in this chunk, added by its first lane
      const unsigned grp = __match_any_sync(0xFFFFFFFFu, in ? sidx : -1 - lane);
      if (in && (__ffs(grp) - 1) == lane) {
        segs[sidx].z += __popc(grp);
      }
      __syncwarp();
      nseg += __popc(sb);
    }
    // T events: the run's new T segments, in order
    for (int j0 = ns0; j0 < nseg; j0 += 32) {
      const int j = j0 + lane;
      const bool is_t = j < nseg && (segs[j].x & 0xFF) == THINKV_T;
      unsigned tb = __ballot_sync(0xFFFFFFFFu, is_t);
      while (tb) {
        const int e = j0 + __ffs(tb) - 1;
        tbe_event(C, T, s, e, t_min, sched, K);
        tb &= tb - 1;
      }
    }
    if (lane < 3) C.free_top[s * 3 + lane] = lane == 0 ? K.top[0] : (lane == 1 ? K.top[1] : K.top[2]);
    if (lane == 0) {
      C.live_count[s] = K.live;
      C.num_live[s] = K.nlive;
      T.nseg[s] = nseg;
    }
  }
}

}  // namespace

cudaError_t launch_tbe(const CacheView& C, int4* seg, int32_t* nseg, int32_t* settled, int32_t n,
                       const int32_t* seq, const int32_t* pos, const uint8_t* tag, int32_t t_min,
                       const int32_t schedule[3], int32_t* run_start, cudaStream_t stream) {
  TbeView T;
  T.seg = seg;
  T.nseg = nseg;
  T.settled = settled;
  const size_t seen_bytes = (size_t)((C.L.max_seqs + 31) / 32) * 4;
  tbe_kernel<<<1, kTbeThreads, seen_bytes, stream>>>(C, T, n, seq, pos, tag, t_min,
                                                     make_int4(schedule[0], schedule[1], schedule[2], 0),
                                                     run_start);
  return cudaGetLastError();
}

}  // namespace thinkv
