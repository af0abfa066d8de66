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
//   compact_assign_kernel (one CTA): validates the call, counts each
//     sequence's live tokens per class by scanning its FIFO windows (the
//     tombstones TBE leaves are skipped), grants pages by block-wide scans,
//     writes dst's tables, FIFOs, live lists, free stacks, slot positions and
//     counters, and lists every moved token's source slot.
//   compact_copy_kernel: one warp per (dst page, kv-head) builds the
//     page-head block in shared memory -- K pieces, V half-words and params of
//     each of its source slots, placed at the new slot -- and writes it out
//     with 16-byte stores.
#include <stdint.h>

#include "thinkv_common.cuh"
#include "thinkv_internal.h"

namespace thinkv {

namespace {

constexpr int kCompactThreads = 1024;
constexpr int kCompactWarps = kCompactThreads / 32;
constexpr int kCopyWarps = 8;

__device__ inline unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

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
  int32_t* tbase;     // [3][n + 1] first moved-token index, per class
  int32_t* src;       // [max_tokens] source pool slot (page * 16 + slot) of each moved token
  int32_t* totals;    // [3] pages granted per class
};

__global__ void __launch_bounds__(kCompactThreads, 1)
    compact_assign_kernel(CacheView S, CacheView Dc, int32_t n, const int32_t* __restrict__ seq,
                          int32_t max_tokens, CompactWs ws) {
  extern __shared__ uint32_t seen[];  // max_seqs bits
  __shared__ int s_err;
  __shared__ int sh[40];
  __shared__ int s_tot[3], s_ttot[3];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int max_seqs = S.L.max_seqs, nb_max = S.L.max_blocks_per_seq;
  const int64_t cap = (int64_t)nb_max * kPage;
  if (tid == 0) s_err = (*S.status != 0 || *Dc.status != 0) ? -1 : 0;
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
  // ---- live tokens per (sequence, class): the FIFO windows without tombstones ----
  for (int i = warp; i < n; i += kCompactWarps) {
    const int s = seq[i];
    for (int c = 0; c < 3; ++c) {
      const int h = S.fifo_head[s * 3 + c], t = S.fifo_tail[s * 3 + c];
      const int32_t* ring = S.fifo + ((int64_t)s * 3 + c) * cap;
      int live = 0;
      for (int k0 = h; k0 < t; k0 += 32)
        live += __popc(__ballot_sync(0xFFFFFFFFu, k0 + lane < t && ring[((int64_t)k0 + lane) % cap] >= 0));
      if (lane == 0) ws.cnt[i * 3 + c] = live;
    }
  }
  __syncthreads();
  // ---- page grants and token offsets in call order, per class ----
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
  // ---- per sequence: dst metadata, and the moved tokens' source slots ----
  for (int i = warp; i < n; i += kCompactWarps) {
    const int s = seq[i];
    const uint64_t* stab = S.block_table + (int64_t)s * nb_max;
    uint64_t* dtab = Dc.block_table + (int64_t)s * nb_max;
    uint64_t* dll = Dc.live_list + (int64_t)s * nb_max;
    int32_t* dli = Dc.live_index + (int64_t)s * nb_max;
    int entry0 = 0, live_total = 0;
    for (int c = 0; c < 3; ++c) {
      const int live = ws.cnt[i * 3 + c];
      const int np = (live + kPage - 1) / kPage;
      const int pb = ws.pbase[c * (n + 1) + i];
      int toff = ws.tbase[c * (n + 1) + i];
      for (int c2 = 0; c2 < c; ++c2) toff += s_ttot[c2];      // class-major token list
      const int h = S.fifo_head[s * 3 + c], t = S.fifo_tail[s * 3 + c];
      const int32_t* ring = S.fifo + ((int64_t)s * 3 + c) * cap;
      int32_t* dring = Dc.fifo + ((int64_t)s * 3 + c) * cap;
      int k = 0;                                              // live tokens so far
      for (int k0 = h; k0 < t; k0 += 32) {
        const int32_t ts = k0 + lane < t ? ring[((int64_t)k0 + lane) % cap] : -1;
        const bool live_t = ts >= 0;
        const unsigned b = __ballot_sync(0xFFFFFFFFu, live_t);
        if (live_t) {
          const int kk = k + __popc(b & lanemask_lt());
          const int page = pb + kk / kPage, slot = kk % kPage, e = entry0 + kk / kPage;
          const uint32_t spage = entry_page(stab[ts >> 4]);
          const int32_t sslot = (int32_t)(spage * kPage + (ts & 15));
          ws.src[toff + kk] = sslot;
          Dc.slot_pos[c][(int64_t)page * kPage + slot] = S.slot_pos[c][sslot];
          dring[kk] = e * kPage + slot;
        }
        k += __popc(b);
      }
      // table entries, live list, unused slots of the last page
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
  if (tid == 0)
    for (int c = 0; c < 3; ++c) {
      ws.totals[c] = s_tot[c];
      Dc.page_bump[c] += s_tot[c];
    }
}

// Copies the bytes of slot `ss` of source block `sb` into slot `ds` of the
// block image `db` (b-bit codes, lane portions interleaved in chunks; see
// include/thinkv.h): K pieces, V half-words, params.  Units of two bytes, one
// per lane, so that pieces of any size and chunk boundaries are handled alike.
__device__ void copy_slot(const uint8_t* sb, int ss, uint8_t* db, int ds, int D, int G, int b) {
  const int lane = threadIdx.x & 31;
  const int NG = D / G;
  const int lane_bytes = D * b / 16;
  const int region = 2 * D * b;                  // bytes of the K (or V) code region
  // K: lane 4*(slot%8)+t holds, per group gr, piece (gr, slot/8) of pb bytes
  const int pb = G * b / 32;
  const int kunits = NG * 4 * (pb / 2);
  for (int u = lane; u < kunits; u += 32) {
    const int hw = u % (pb / 2), t = (u / (pb / 2)) % 4, gr = u / (pb / 2) / 4;
    const int so = lane_off(4 * (ss & 7) + t, (gr * 2 + (ss >> 3)) * pb + 2 * hw, lane_bytes);
    const int dof = lane_off(4 * (ds & 7) + t, (gr * 2 + (ds >> 3)) * pb + 2 * hw, lane_bytes);
    *reinterpret_cast<uint16_t*>(db + dof) = *reinterpret_cast<const uint16_t*>(sb + so);
  }
  // V: word (P, q) of lane 4g + t holds slots 2t + 8P (low half) and 2t + 8P + 1 (high half)
  const int Q = b == 16 ? D / 8 : D * b / 128;
  for (int u = lane; u < 8 * Q; u += 32) {
    const int g = u / Q, q = u % Q;
    const int so = lane_off(4 * g + ((ss & 7) >> 1), ((ss >> 3) * Q + q) * 4 + 2 * (ss & 1), lane_bytes);
    const int dof = lane_off(4 * g + ((ds & 7) >> 1), ((ds >> 3) * Q + q) * 4 + 2 * (ds & 1), lane_bytes);
    *reinterpret_cast<uint16_t*>(db + region + dof) =
        *reinterpret_cast<const uint16_t*>(sb + region + so);
  }
  if (b < 16) {
    // params: [K|V][group][slot][scale, zero]
    for (int u = lane; u < 2 * NG; u += 32) {
      const int kv = u / NG, gr = u % NG;
      const int base = 2 * region + kv * 64 * NG;
      *reinterpret_cast<uint32_t*>(db + base + (gr * 16 + ds) * 4) =
          *reinterpret_cast<const uint32_t*>(sb + base + (gr * 16 + ss) * 4);
    }
  }
}

__global__ void __launch_bounds__(kCopyWarps * 32)
    compact_copy_kernel(CacheView S, CacheView Dc, int32_t n, CompactWs ws, int max_phb) {
  extern __shared__ __align__(16) uint8_t img[];   // kCopyWarps block images
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
    // the call index whose pages hold dst page (page_bump at the call) + gp
    const int32_t* pb = ws.pbase + c * (n + 1);
    const int page = pb[0] + gp;
    int lo = 0, hi = n;                             // last i with pb[i] <= page
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (pb[mid] <= page) lo = mid; else hi = mid;
    }
    const int i = lo;
    const int live = ws.cnt[i * 3 + c];
    const int j = page - pb[i];                     // page of the sequence's class-c run
    const int used = min(kPage, live - j * kPage);
    int toff = ws.tbase[c * (n + 1) + i] + j * kPage;
    for (int c2 = 0; c2 < c; ++c2) toff += ws.tbase[c2 * (n + 1) + n];
    for (int sl = 0; sl < used; ++sl) {
      const int32_t src = ws.src[toff + sl];
      const uint8_t* sb = S.pool[c] + ((int64_t)(src >> 4) * H + h) * phb;
      copy_slot(sb, src & 15, db, sl, D, G, b);
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
  compact_assign_kernel<<<1, kCompactThreads, seen_bytes, stream>>>(S, Dc, n, seq, max_tokens, ws);
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
