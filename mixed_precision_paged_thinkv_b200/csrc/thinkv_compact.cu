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
//     page-head block in shared memory -- K pieces, V half-words and params of
//     each of its source slots at the new slot, every two-byte unit a load of
//     its own, all in flight together -- and writes it out with 16-byte stores.
#include <stdint.h>

#include "thinkv_common.cuh"
#include "thinkv_internal.h"

namespace thinkv {

namespace {

constexpr int kCompactThreads = 1024;
constexpr int kCompactWarps = kCompactThreads / 32;
constexpr int kCopyWarps = 8;

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

// Byte offsets of unit u (two bytes) of one slot's data inside a page-head
// block (b-bit codes, lane portions interleaved in chunks; include/thinkv.h):
// units [0, ku) are K pieces, [ku, ku + kv) V half-words, then params words
// (counted as two units each).
struct SlotUnits {
  int D, G, b, NG, lane_bytes, region, pb, ku, kvu, Q;
};

__device__ inline SlotUnits slot_units(int D, int G, int b) {
  SlotUnits m;
  m.D = D; m.G = G; m.b = b; m.NG = D / G;
  m.lane_bytes = D * b / 16;
  m.region = 2 * D * b;
  m.pb = G * b / 32;
  m.ku = m.NG * 4 * (m.pb / 2);
  m.Q = b == 16 ? D / 8 : D * b / 128;
  m.kvu = 8 * m.Q;
  return m;
}

// source and destination offsets (and size, 2 or 4) of unit u of slot ss -> ds
__device__ inline int unit_offsets(const SlotUnits& m, int u, int ss, int ds, int* so, int* dof) {
  if (u < m.ku) {
    const int hw = u % (m.pb / 2), t = (u / (m.pb / 2)) % 4, gr = u / (m.pb / 2) / 4;
    *so = lane_off(4 * (ss & 7) + t, (gr * 2 + (ss >> 3)) * m.pb + 2 * hw, m.lane_bytes);
    *dof = lane_off(4 * (ds & 7) + t, (gr * 2 + (ds >> 3)) * m.pb + 2 * hw, m.lane_bytes);
    return 2;
  }
  u -= m.ku;
  if (u < m.kvu) {
    const int g = u / m.Q, q = u % m.Q;
    *so = m.region + lane_off(4 * g + ((ss & 7) >> 1), ((ss >> 3) * m.Q + q) * 4 + 2 * (ss & 1), m.lane_bytes);
    *dof = m.region + lane_off(4 * g + ((ds & 7) >> 1), ((ds >> 3) * m.Q + q) * 4 + 2 * (ds & 1), m.lane_bytes);
    return 2;
  }
  u -= m.kvu;                                      // params: [K|V][group][slot] words
  const int kv = u / m.NG, gr = u % m.NG;
  const int base = 2 * m.region + kv * 64 * m.NG;
  *so = base + (gr * 16 + ss) * 4;
  *dof = base + (gr * 16 + ds) * 4;
  return 4;
}

// (d) one warp per (dst page, kv-head): the page-head block is gathered into
// shared memory -- every unit of every slot a lane load of its own, all in
// flight together -- and written out with 16-byte stores
__global__ void __launch_bounds__(kCopyWarps * 32)
    compact_copy_kernel(CacheView S, CacheView Dc, int32_t n, CompactWs ws, int max_phb) {
  extern __shared__ __align__(16) uint8_t img[];   // kCopyWarps block images
  if (ws.totals[3] == 0) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int H = S.L.num_kv_heads, D = S.L.head_dim, G = S.L.group_size;
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
    const SlotUnits m = slot_units(D, G, b);
    const int per = m.ku + m.kvu + 2 * m.NG;
    for (int x0 = 0; x0 < used * per; x0 += 32) {     // warp-uniform trip count
      const int x = x0 + lane;
      const int sl = min(x / per, used - 1), uu = x - sl * per;
      const int32_t src = __shfl_sync(0xFFFFFFFFu, srcl, sl);
      if (x < used * per) {
        int so, dof;
        const int sz = unit_offsets(m, uu, src & 15, sl, &so, &dof);
        const uint8_t* sb = S.pool[c] + ((int64_t)(src >> 4) * H + h) * phb;
        if (sz == 2) *reinterpret_cast<uint16_t*>(db + dof) = *reinterpret_cast<const uint16_t*>(sb + so);
        else *reinterpret_cast<uint32_t*>(db + dof) = *reinterpret_cast<const uint32_t*>(sb + so);
      }
    }
    __syncwarp();
    uint4* dst = reinterpret_cast<uint4*>(Dc.pool[c] + ((int64_t)page * H + h) * phb);
    for (int x = lane; x < phb / 16; x += 32) dst[x] = reinterpret_cast<const uint4*>(db)[x];
    __syncwarp();
  }
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
  const size_t smem = (size_t)kCopyWarps * max_phb;
  if (smem > 48 * 1024) {
    e = cudaFuncSetAttribute(compact_copy_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
  }
  compact_copy_kernel<<<num_sms * 4, kCopyWarps * 32, smem, stream>>>(S, Dc, n, ws, max_phb);
  return cudaGetLastError();
}

}  // namespace thinkv
