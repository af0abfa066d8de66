// thinkv_compact.cu -- gather compaction: the step Continuous Thinking avoids.
//
// "ThinKV: Thought-Adaptive KV Cache Compression for Efficient Reasoning
// Models", explainer, Methodologie, "Implementation Systeme: Pensee Continue
// (CT)": evicting scattered tokens leaves holes; the usual remedy is a
// gather-based compaction that moves the survivors together, at a cost in
// time and HBM bandwidth (Resultats: the TPOT gain comes mainly from not
// compacting).  CT refills holes in place instead.  This kernel pair is that
// compaction, built so that what CT saves can be measured on the same states.
//
// Reading: each listed sequence's live tokens move into fresh hole-free pages
// of an empty cache `dst` of the same geometry -- class by class (R, E, T),
// FIFO (arrival) order within a class, 16 to a page -- as if appended there in
// that order with their codes copied, not requantised; the last page of a
// class keeps its unused slots on the free stack.  Pages are granted in call
// order per class.
//
//   compact_count_kernel: a warp per (sequence, class) counts the live tokens
//     of its FIFO window (TBE's tombstones skipped), 256 entries in flight.
//   compact_plan_kernel (one CTA): validates the call, grants pages and token
//     offsets by block-wide scans in call order, and writes the destination's
//     tables, live lists, free stacks, counters and the unused slots of each
//     last page; a flag tells the next kernels that the plan succeeded.
//   compact_list_kernel: a warp per (sequence, class) walks the FIFO window
//     again and writes every moved token's source slot, destination FIFO
//     entry and slot position.
//   compact_copy_kernel: one warp per (dst page, kv-head) gathers the
//     page-head block in shared memory -- each source slot's K pieces (whole,
//     up to 16 bytes), V half-words and params words at the new slot, a load
//     per unit, sixteen per lane in flight -- and writes it out with 16-byte
//     stores.
#include <stdint.h>

#include "thinkv_common.cuh"
#include "thinkv_internal.h"

namespace thinkv {

namespace {

constexpr int kCompactThreads = 1024;
constexpr int kCompactWarps = kCompactThreads / 32;
constexpr int kCopyWarps = 8;
constexpr int kCopyBlocks = 2;    // resident copy CTAs per SM (128 registers)
// gather loads in flight per lane (compact_copy_kernel): 8 narrow units, or
// 64 bytes of 8- and 16-byte units
template <int N> __host__ __device__ constexpr int copy_batch() { return N >= 8 ? 64 / N : 8; }

// Block-wide exclusive scan (kCompactThreads threads) of one int per thread.
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
    int w = lane < kCompactWarps ? sh[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xFFFFFFFFu, w, o);
      if (lane >= o) w += y;
    }
    sh[lane] = w;
  }
  __syncthreads();
  const int excl = (warp == 0 ? 0 : sh[warp - 1]) + x - v;
  *total = sh[kCompactWarps - 1];
  __syncthreads();
  return excl;
}

struct CompactWs {
  int32_t* cnt;       // [n][3] live tokens per (call index, class)
  int32_t* pbase;     // [3][n + 1] first dst page of each call index, per class
  int32_t* tbase;     // [3][n + 1] first moved-token index, per class (class-major list)
  int32_t* src;       // [max_tokens] source pool slot (page * 16 + slot) of each moved token
  int32_t* totals;    // [3] pages granted per class; [3]: 1 once the plan succeeded
};

constexpr int kScan = 8;     // FIFO entries per lane per pass (loads in flight)

// FIFO entries [k0, k0 + 32 * kScan) of a ring, kScan per lane in lane-major
// order (entry k0 + lane * kScan + j); entries at or past t read as -1.
__device__ inline void load_fifo(const int32_t* ring, int64_t cap, int k0, int t,
                                 int32_t (&x)[kScan]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int j = 0; j < kScan; ++j) {
    const int k = k0 + lane * kScan + j;
    x[j] = k < t ? ring[(int64_t)k % cap] : -1;
  }
}

// (a) live tokens of each (call index, class): a warp per pair, kScan entries per lane in flight
__global__ void compact_count_kernel(CacheView S, int32_t n, const int32_t* __restrict__ seq,
                                     CompactWs ws) {
  const int lane = threadIdx.x & 31;
  const int64_t cap = (int64_t)S.L.max_blocks_per_seq * kPage;
  const int64_t gw = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t x = gw; x < (int64_t)n * 3; x += nw) {
    const int i = (int)(x / 3), c = (int)(x % 3);
    const int s = seq[i];
    int live = 0;
    if (s >= 0 && s < S.L.max_seqs) {
      const int h = S.fifo_head[s * 3 + c], t = S.fifo_tail[s * 3 + c];
      const int32_t* ring = S.fifo + ((int64_t)s * 3 + c) * cap;
      for (int k0 = h; k0 < t; k0 += 32 * kScan) {
        int32_t e[kScan];
        load_fifo(ring, cap, k0, t, e);
#pragma unroll
        for (int j = 0; j < kScan; ++j) live += e[j] >= 0;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) live += __shfl_xor_sync(0xFFFFFFFFu, live, o);
    }
    if (lane == 0) ws.cnt[x] = live;
  }
}

// (b) one CTA: validation, page grants and token offsets in call order, and
// each sequence's destination metadata that follows from the counts alone
__global__ void __launch_bounds__(kCompactThreads, 1)
    compact_plan_kernel(CacheView S, CacheView Dc, int32_t n, const int32_t* __restrict__ seq,
                        int32_t max_tokens, CompactWs ws) {
  extern __shared__ uint32_t seen[];  // max_seqs bits
  __shared__ int s_err;
  __shared__ int sh[40];
  __shared__ int s_tot[3], s_ttot[3];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int max_seqs = S.L.max_seqs, nb_max = S.L.max_blocks_per_seq;
  const int64_t cap = (int64_t)nb_max * kPage;
  if (tid == 0) {
    s_err = (*S.status != 0 || *Dc.status != 0) ? -1 : 0;
    ws.totals[3] = 0;
  }
  for (int i = tid; i < (max_seqs + 31) / 32; i += kCompactThreads) seen[i] = 0;
  __syncthreads();
  if (s_err != 0) return;
  for (int i = tid; i < n; i += kCompactThreads) {
    const int s = seq[i];
    bool bad = s < 0 || s >= max_seqs;
    if (!bad) {
      const uint32_t old = atomicOr(&seen[s >> 5], 1u << (s & 31));
      bad = (old & (1u << (s & 31))) || Dc.num_blocks[s] != 0;   // distinct; dst empty for s
    }
    if (bad) s_err = THINKV_ERR_INVALID;
  }
  __syncthreads();
  if (s_err != 0) {
    if (tid == 0) set_status(Dc.status, s_err);
    return;
  }
  for (int c = 0; c < 3; ++c) {
    int pcarry = 0, tcarry = 0;
    for (int base = 0; base < n; base += kCompactThreads) {
      const int i = base + tid;
      const int live = i < n ? ws.cnt[i * 3 + c] : 0;
      int ptot, ttot;
      const int pex = block_scan((live + kPage - 1) / kPage, sh, &ptot);
      const int tex = block_scan(live, sh, &ttot);
      if (i < n) {
        ws.pbase[c * (n + 1) + i] = Dc.page_bump[c] + pcarry + pex;
        ws.tbase[c * (n + 1) + i] = tcarry + tex;
      }
      pcarry += ptot;
      tcarry += ttot;
    }
    if (tid == 0) {
      s_tot[c] = pcarry;
      s_ttot[c] = tcarry;
      ws.pbase[c * (n + 1) + n] = Dc.page_bump[c] + pcarry;
      ws.tbase[c * (n + 1) + n] = tcarry;
    }
  }
  __syncthreads();
  if (tid == 0) {
    int err = 0;
    for (int c = 0; c < 3; ++c)
      if ((int64_t)Dc.page_bump[c] + s_tot[c] > Dc.L.pool_pages[c]) err = THINKV_ERR_OUT_OF_PAGES;
    if ((int64_t)s_ttot[0] + s_ttot[1] + s_ttot[2] > max_tokens) err = THINKV_ERR_INVALID;
    s_err = err;
    if (err) set_status(Dc.status, err);
  }
  __syncthreads();
  if (s_err != 0) return;
  for (int i = warp; i < n; i += kCompactWarps) {
    const int s = seq[i];
    uint64_t* dtab = Dc.block_table + (int64_t)s * nb_max;
    uint64_t* dll = Dc.live_list + (int64_t)s * nb_max;
    int32_t* dli = Dc.live_index + (int64_t)s * nb_max;
    int entry0 = 0, live_total = 0;
    for (int c = 0; c < 3; ++c) {
      const int live = ws.cnt[i * 3 + c];
      const int np = (live + kPage - 1) / kPage;
      const int pb = ws.pbase[c * (n + 1) + i];
      for (int j = lane; j < np; j += 32) {
        const int used = min(kPage, live - j * kPage);
        const uint32_t mask = used >= kPage ? 0xFFFFu : ((1u << used) - 1u);
        const int e = entry0 + j;
        dtab[e] = make_entry((uint32_t)(pb + j), c, mask);
        dll[e] = make_live_desc((uint32_t)(pb + j), c, e);
        dli[e] = e;
        if (j == np - 1)
          for (int sl = used; sl < kPage; ++sl) Dc.slot_pos[c][(int64_t)(pb + j) * kPage + sl] = -1;
      }
      const int used_last = live - (np - 1) * kPage;
      const int nfree = np > 0 ? kPage - used_last : 0;
      int32_t* dstack = Dc.free_slots + ((int64_t)s * 3 + c) * cap;
      for (int x = lane; x < nfree; x += 32) dstack[x] = (entry0 + np - 1) * kPage + (kPage - 1 - x);
      if (lane == 0) {
        Dc.free_top[s * 3 + c] = nfree;
        Dc.fifo_head[s * 3 + c] = 0;
        Dc.fifo_tail[s * 3 + c] = live;
      }
      entry0 += np;
      live_total += live;
    }
    if (lane == 0) {
      Dc.num_blocks[s] = entry0;
      Dc.num_live[s] = entry0;
      Dc.live_count[s] = live_total;
    }
  }
  __syncthreads();
  if (tid == 0) {
    for (int c = 0; c < 3; ++c) {
      ws.totals[c] = s_tot[c];
      Dc.page_bump[c] += s_tot[c];
    }
    ws.totals[3] = 1;
  }
}

// (c) the moved tokens in order: a warp per (call index, class) walks the
// source FIFO window and writes each live token's source slot, its
// destination FIFO entry and slot position
__global__ void compact_list_kernel(CacheView S, CacheView Dc, int32_t n,
                                    const int32_t* __restrict__ seq, CompactWs ws) {
  if (ws.totals[3] == 0) return;                 // the plan failed: nothing moves
  const int lane = threadIdx.x & 31;
  const int nb_max = S.L.max_blocks_per_seq;
  const int64_t cap = (int64_t)nb_max * kPage;
  const int64_t gw = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t x = gw; x < (int64_t)n * 3; x += nw) {
    const int i = (int)(x / 3), c = (int)(x % 3);
    const int s = seq[i];
    const uint64_t* stab = S.block_table + (int64_t)s * nb_max;
    int entry0 = 0;                               // pages of the earlier classes of s
    for (int c2 = 0; c2 < c; ++c2) entry0 += (ws.cnt[i * 3 + c2] + kPage - 1) / kPage;
    const int pb = ws.pbase[c * (n + 1) + i];
    int toff = ws.tbase[c * (n + 1) + i];
    for (int c2 = 0; c2 < c; ++c2) toff += ws.tbase[c2 * (n + 1) + n];
    const int h = S.fifo_head[s * 3 + c], t = S.fifo_tail[s * 3 + c];
    const int32_t* ring = S.fifo + ((int64_t)s * 3 + c) * cap;
    int32_t* dring = Dc.fifo + ((int64_t)s * 3 + c) * cap;
    int k = 0;                                    // live tokens before this pass
    for (int k0 = h; k0 < t; k0 += 32 * kScan) {
      int32_t e[kScan];
      load_fifo(ring, cap, k0, t, e);
      int mine = 0;
#pragma unroll
      for (int j = 0; j < kScan; ++j) mine += e[j] >= 0;
      int before = mine;                          // exclusive prefix over lanes
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xFFFFFFFFu, before, o);
        if (lane >= o) before += y;
      }
      const int total = __shfl_sync(0xFFFFFFFFu, before, 31);
      int kk = k + before - mine;
#pragma unroll
      for (int j = 0; j < kScan; ++j) {
        if (e[j] < 0) continue;
        const int page = pb + kk / kPage, slot = kk % kPage, ent = entry0 + kk / kPage;
        const int32_t sslot = (int32_t)(entry_page(stab[e[j] >> 4]) * kPage + (e[j] & 15));
        ws.src[toff + kk] = sslot;
        Dc.slot_pos[c][(int64_t)page * kPage + slot] = S.slot_pos[c][sslot];
        dring[kk] = ent * kPage + slot;
        ++kk;
      }
      k += total;
    }
  }
}

// Byte offsets of unit u of one slot's data inside a page-head block of
// b-bit codes (lane portions interleaved in chunks; include/thinkv.h): units
// [0, KU) are two-byte K pieces, [KU, KU + KVU) V half-words, then (b < 16)
// the four-byte (scale, zero) words of K and V per group.  All shapes are
// compile-time, so every divide is a shift.
template <int D, int G, int B>
struct SlotUnits {
  static constexpr int NG = D / G;
  static constexpr int LB = D * B / 16;                 // lane portion bytes
  static constexpr int REGION = 2 * D * B;
  static constexpr int PB = G * B / 32;                 // K piece bytes
  static constexpr int HW = PB / 2;                     // two-byte units per piece
  static constexpr int KU = NG * 4 * HW;
  static constexpr int Q = B == 16 ? D / 8 : D * B / 128;
  static constexpr int KVU = 8 * Q;
  static constexpr int PHB = B == 16 ? 64 * D : 4 * D * B + 128 * NG;
  static constexpr int CH = LB < 16 ? LB : 16;          // chunk bytes

  __device__ static int lane_at(int l, int o) { return (o / CH) * 32 * CH + l * CH + (o % CH); }

  // source and destination offsets of unit u of slot ss -> ds; returns the size (2 or 4)
  __device__ static int offsets(int u, int ss, int ds, int* so, int* dof) {
    if (u < KU) {
      const int hw = u % HW, t = (u / HW) % 4, gr = u / HW / 4;
      *so = lane_at(4 * (ss & 7) + t, (gr * 2 + (ss >> 3)) * PB + 2 * hw);
      *dof = lane_at(4 * (ds & 7) + t, (gr * 2 + (ds >> 3)) * PB + 2 * hw);
      return 2;
    }
    u -= KU;
    if (u < KVU) {
      const int g = u / Q, q = u % Q;
      *so = REGION + lane_at(4 * g + ((ss & 7) >> 1), ((ss >> 3) * Q + q) * 4 + 2 * (ss & 1));
      *dof = REGION + lane_at(4 * g + ((ds & 7) >> 1), ((ds >> 3) * Q + q) * 4 + 2 * (ds & 1));
      return 2;
    }
    u -= KVU;                                          // params: [K|V][group][slot] words
    const int kv = u / NG, gr = u % NG;
    const int base = 2 * REGION + kv * 64 * NG;
    *so = base + (gr * 16 + ss) * 4;
    *dof = base + (gr * 16 + ds) * 4;
    return 4;
  }
};

// Loads and stores of one unit of N bytes (N = 2, 4, 8 or 16).
template <int N> struct UnitT;
template <> struct UnitT<2> { using T = uint16_t; };
template <> struct UnitT<4> { using T = uint32_t; };
template <> struct UnitT<8> { using T = uint2; };
template <> struct UnitT<16> { using T = uint4; };

// Copies `total` units of N bytes into the warp's image db, lane-strided,
// copy_batch<N>() loads in flight per lane before their stores.  at(x, &so, &dof,
// &sb) gives unit x's source block, source offset and image offset.
template <int N, typename At>
__device__ __forceinline__ void gather_units(int total, uint8_t* db, At at) {
  using T = typename UnitT<N>::T;
  constexpr int NB = copy_batch<N>();
  const int lane = threadIdx.x & 31;
  for (int x0 = 0; x0 < total; x0 += 32 * NB) {     // warp-uniform trip count
    T val[NB];
    int dst[NB];                                  // image offset; -1: none
#pragma unroll
    for (int j = 0; j < NB; ++j) {
      const int x = x0 + j * 32 + lane;
      int so = 0, dof = -1;
      const uint8_t* sb = nullptr;
      at(x < total ? x : total - 1, &so, &dof, &sb);   // shuffles inside: every lane takes part
      dst[j] = x < total ? dof : -1;
      if (x < total) val[j] = *reinterpret_cast<const T*>(sb + so);
    }
#pragma unroll
    for (int j = 0; j < NB; ++j)
      if (dst[j] >= 0) *reinterpret_cast<T*>(db + dst[j]) = val[j];
  }
}

// One page-head block gathered into the warp's shared-memory image db.  K
// moves as whole pieces (units of up to 16 bytes: a piece never straddles a
// chunk), then V half-words and (b < 16) the params words.  srcl: lane sl
// holds slot sl's source pool slot (page * 16 + slot).
template <int D, int G, int B>
__device__ __forceinline__ void gather_block(const uint8_t* __restrict__ pool, int H, int h, int32_t srcl, int used,
                             uint8_t* db) {
  using M = SlotUnits<D, G, B>;
  constexpr int KPU = M::PB < 16 ? M::PB : 16;          // K unit bytes
  constexpr int KPN = M::PB / KPU;                      // units per piece
  constexpr int KPER = 4 * M::NG * KPN;                 // K units per slot
  auto src_of = [&](int sl, int* ss, const uint8_t** sb) {
    const int32_t src = __shfl_sync(0xFFFFFFFFu, srcl, sl);
    *ss = src & 15;
    *sb = pool + ((int64_t)(src >> 4) * H + h) * M::PHB;
  };
  gather_units<KPU>(used * KPER, db, [&](int x, int* so, int* dof, const uint8_t** sb) {
    const int sl = x / KPER, u = x - sl * KPER;
    int ss;
    src_of(sl, &ss, sb);
    const int kp = u % KPN, t = (u / KPN) % 4, gr = u / KPN / 4;
    *so = M::lane_at(4 * (ss & 7) + t, (gr * 2 + (ss >> 3)) * M::PB + kp * KPU);
    *dof = M::lane_at(4 * (sl & 7) + t, (gr * 2 + (sl >> 3)) * M::PB + kp * KPU);
  });
  // V half-words (2 bytes) and params words (4 bytes): two passes of one width each
  gather_units<2>(used * M::KVU, db, [&](int x, int* so, int* dof, const uint8_t** sb) {
    const int sl = x / M::KVU, u = x - sl * M::KVU;
    int ss;
    src_of(sl, &ss, sb);
    M::offsets(M::KU + u, ss, sl, so, dof);
  });
  if constexpr (B < 16) {
    constexpr int PU = 2 * M::NG;                       // params words per slot
    gather_units<4>(used * PU, db, [&](int x, int* so, int* dof, const uint8_t** sb) {
      const int sl = x / PU, u = x - sl * PU;
      int ss;
      src_of(sl, &ss, sb);
      M::offsets(M::KU + M::KVU + u, ss, sl, so, dof);
    });
  }
}

template <int D, int G>
__device__ inline void gather_dispatch(int b, const uint8_t* pool, int H, int h, int32_t srcl,
                                       int used, uint8_t* db) {
  switch (b) {
    case 2: gather_block<D, G, 2>(pool, H, h, srcl, used, db); break;
    case 4: gather_block<D, G, 4>(pool, H, h, srcl, used, db); break;
    case 8: gather_block<D, G, 8>(pool, H, h, srcl, used, db); break;
    default: gather_block<D, G, 16>(pool, H, h, srcl, used, db); break;
  }
}

// (d) one warp per (dst page, kv-head): the page-head block is gathered into
// shared memory (gather_block) and written out with 16-byte stores
template <int D, int G>
__global__ void __launch_bounds__(kCopyWarps * 32, kCopyBlocks)
    compact_copy_kernel(CacheView S, CacheView Dc, int32_t n, CompactWs ws, int max_phb) {
  extern __shared__ __align__(16) uint8_t img[];   // kCopyWarps block images
  if (ws.totals[3] == 0) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int H = S.L.num_kv_heads;
  const int t0 = ws.totals[0], t1 = ws.totals[1], t2 = ws.totals[2];
  const int64_t units = (int64_t)(t0 + t1 + t2) * H;
  uint8_t* db = img + warp * max_phb;
  for (int64_t u = (int64_t)blockIdx.x * kCopyWarps + warp; u < units;
       u += (int64_t)gridDim.x * kCopyWarps) {
    const int h = (int)(u % H);
    int gp = (int)(u / H);                          // dst page over the classes
    const int c = gp < t0 ? 0 : (gp < t0 + t1 ? 1 : 2);
    gp -= c == 0 ? 0 : (c == 1 ? t0 : t0 + t1);
    const int b = S.L.bits[c];
    const int phb = (int)page_head_bytes(D, G, b);
    const int32_t* pb = ws.pbase + c * (n + 1);
    const int page = pb[0] + gp;
    int lo = 0, hi = n;                             // last i with pb[i] <= page
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (pb[mid] <= page) lo = mid; else hi = mid;
    }
    const int i = lo;
    const int live = ws.cnt[i * 3 + c];
    const int j = page - pb[i];
    const int used = min(kPage, live - j * kPage);
    int toff = ws.tbase[c * (n + 1) + i] + j * kPage;
    for (int c2 = 0; c2 < c; ++c2) toff += ws.tbase[c2 * (n + 1) + n];
    const int32_t srcl = lane < used ? ws.src[toff + lane] : 0;   // lane sl: slot sl's source
    gather_dispatch<D, G>(b, S.pool[c], H, h, srcl, used, db);
    __syncwarp();
    uint4* dst = reinterpret_cast<uint4*>(Dc.pool[c] + ((int64_t)page * H + h) * phb);
    for (int x = lane; x < phb / 16; x += 32) dst[x] = reinterpret_cast<const uint4*>(db)[x];
    __syncwarp();
  }
}

template <int D, int G>
cudaError_t launch_copy(const CacheView& S, const CacheView& Dc, int32_t n, const CompactWs& ws,
                        int max_phb, int num_sms, cudaStream_t stream) {
  const size_t smem = (size_t)kCopyWarps * max_phb;
  if (smem > 48 * 1024) {
    const cudaError_t e = cudaFuncSetAttribute(compact_copy_kernel<D, G>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  compact_copy_kernel<D, G><<<num_sms * kCopyBlocks, kCopyWarps * 32, smem, stream>>>(S, Dc, n, ws,
                                                                                  max_phb);
  return cudaGetLastError();
}

}  // namespace

size_t compact_workspace_bytes(int32_t n, int32_t max_tokens) {
  auto r = [](size_t x) { return (x + 255) / 256 * 256; };
  return r((size_t)n * 3 * 4) + 2 * r((size_t)3 * (n + 1) * 4) + r((size_t)max_tokens * 4) + 256;
}

cudaError_t launch_compact(const CacheView& S, const CacheView& Dc, int32_t n, const int32_t* seq,
                           int32_t max_tokens, void* workspace, int num_sms, cudaStream_t stream) {
  auto r = [](size_t x) { return (x + 255) / 256 * 256; };
  uint8_t* w = static_cast<uint8_t*>(workspace);
  CompactWs ws;
  ws.cnt = reinterpret_cast<int32_t*>(w);
  w += r((size_t)n * 3 * 4);
  ws.pbase = reinterpret_cast<int32_t*>(w);
  w += r((size_t)3 * (n + 1) * 4);
  ws.tbase = reinterpret_cast<int32_t*>(w);
  w += r((size_t)3 * (n + 1) * 4);
  ws.src = reinterpret_cast<int32_t*>(w);
  w += r((size_t)max_tokens * 4);
  ws.totals = reinterpret_cast<int32_t*>(w);
  const size_t seen_bytes = (size_t)((S.L.max_seqs + 31) / 32) * 4;
  const int64_t pairs = (int64_t)n * 3;
  const int gblocks = (int)((pairs * 32 + 255) / 256);
  if (seen_bytes > 48 * 1024) {
    const cudaError_t a = cudaFuncSetAttribute(compact_plan_kernel,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)seen_bytes);
    if (a != cudaSuccess) return a;
  }
  compact_count_kernel<<<gblocks, 256, 0, stream>>>(S, n, seq, ws);
  compact_plan_kernel<<<1, kCompactThreads, seen_bytes, stream>>>(S, Dc, n, seq, max_tokens, ws);
  compact_list_kernel<<<gblocks, 256, 0, stream>>>(S, Dc, n, seq, ws);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  int max_phb = 0;
  for (int c = 0; c < 3; ++c) {
    const int b = (int)page_head_bytes(S.L.head_dim, S.L.group_size, S.L.bits[c]);
    max_phb = b > max_phb ? b : max_phb;
  }
  const int D = S.L.head_dim, G = S.L.group_size;
  if (D == 128 && G == 64) return launch_copy<128, 64>(S, Dc, n, ws, max_phb, num_sms, stream);
  if (D == 128 && G == 32) return launch_copy<128, 32>(S, Dc, n, ws, max_phb, num_sms, stream);
  if (D == 64 && G == 64) return launch_copy<64, 64>(S, Dc, n, ws, max_phb, num_sms, stream);
  return launch_copy<64, 32>(S, Dc, n, ws, max_phb, num_sms, stream);
}

}  // namespace thinkv
