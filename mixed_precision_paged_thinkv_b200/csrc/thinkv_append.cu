// thinkv_append.cu -- quantize-on-append into reused slots (TBQ + CT write path).
//
// "ThinKV: Thought-Adaptive KV Cache Compression for Efficient Reasoning
// Models", explainer, Methodologie: TBQ gives each token the precision of its
// thought type (R > E > T) by group quantisation; "Implementation Systeme:
// Pensee Continue (CT)" lets a new token of a thought type overwrite a slot
// freed by eviction, so the cache is never compacted.
//
// Two launches:
//   1. append_assign_kernel (one CTA): validates the call, counts per-(sequence,
//      class) demand, grants pages in call order with block-wide exclusive
//      scans, then one warp per sequence run pops free slots / opens pages,
//      writes table entries, slot positions, FIFO pushes, live-list joins and
//      the final free stacks.  It writes every token's pool slot id to the
//      workspace, and a go/no-go flag (the call is all-or-nothing).
//   2. append_scatter_kernel (grid): one warp per (token, kv-head, K|V):
//      group min/max by warp shuffles, directed-rounded fp16 zero/scale,
//      round-half-even codes, then scatter into the page-head block (lane
//      portions interleaved in 16-byte chunks).
#include <cuda_fp16.h>
#include <stdint.h>

#include "thinkv_common.cuh"
#include "thinkv_evict_seq.cuh"
#include "thinkv_internal.h"

namespace thinkv {

namespace {

constexpr int kAssignThreads = 1024;
constexpr int kSmallAppend = 512;   // calls of at most this many tokens take the one-launch path
constexpr int kAssignWarps = kAssignThreads / 32;

__device__ inline unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Block-wide exclusive scan of one int per thread (1024 threads); returns the
// exclusive prefix, `total` gets the block sum.  Uses `sh` (>= 33 ints).
__device__ int block_exclusive_scan(int v, int* sh, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xFFFFFFFFu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sh[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = lane < kAssignWarps ? sh[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xFFFFFFFFu, w, o);
      if (lane >= o) w += y;
    }
    sh[lane] = w;  // inclusive warp prefix
  }
  __syncthreads();
  int warp_excl = warp == 0 ? 0 : sh[warp - 1];
  *total = sh[kAssignWarps - 1];
  __syncthreads();
  return warp_excl + x - v;
}

// Slot assignment of one sequence run (one warp): tokens start..start+len-1
// of sequence s, cnt[c] tokens of class c, new pages of class c numbered from
// page_base[c] on.  Each token takes the top of its (sequence, class) free
// stack, or the next slot of a new page; table entries, slot positions, FIFO
// pushes, live-list joins, the final free stacks and the sequence counters
// are written, and tok_slot[i] gets token i's pool slot (page * 16 + slot).
// Only this warp touches sequence s's state during the call.  `st`, if not
// null, holds s's counters already loaded: free_top[3], fifo_tail[3],
// num_blocks, num_live, live_count.
__device__ void assign_run(const CacheView& C, int s, int start, int len, const int (&cnt_in)[3],
                           const int (&page_base)[3], const int32_t* __restrict__ pos,
                           const uint8_t* __restrict__ tag, int32_t* tok_slot,
                           const int* st = nullptr) {
  const int lane = threadIdx.x & 31;
  const int nb_max = C.L.max_blocks_per_seq;
  const int64_t cap = (int64_t)nb_max * kPage;
  uint64_t* table = C.block_table + (int64_t)s * nb_max;
  uint64_t* llist = C.live_list + (int64_t)s * nb_max;
  int32_t* lidx = C.live_index + (int64_t)s * nb_max;
  int F[3], tail[3], rank[3] = {0, 0, 0}, last_entry[3] = {-1, -1, -1};
#pragma unroll
  for (int cc = 0; cc < 3; ++cc) {
    F[cc] = st ? st[cc] : C.free_top[s * 3 + cc];
    tail[cc] = st ? st[3 + cc] : C.fifo_tail[s * 3 + cc];
  }
  const int nb0 = st ? st[6] : C.num_blocks[s];
  int grants = 0;
  int nlive = st ? st[7] : C.num_live[s];
  for (int base = start; base < start + len; base += 32) {
    const int i = base + lane;
    const bool valid = i < start + len;
    const int c = valid ? tag[i] : 0;
    unsigned bal[3], gbal_c[3];
#pragma unroll
    for (int cc = 0; cc < 3; ++cc) bal[cc] = __ballot_sync(0xFFFFFFFFu, valid && c == cc);
    const int k = rank[c] + __popc(bal[c] & lanemask_lt());
    const bool is_pop = valid && k < F[c];
    const int kp = k - F[c];
    const int j = kp >> 4, slot_new = kp & 15;
    const bool is_grant = valid && !is_pop && slot_new == 0;
#pragma unroll
    for (int cc = 0; cc < 3; ++cc) gbal_c[cc] = __ballot_sync(0xFFFFFFFFu, is_grant && c == cc);
    const unsigned gbal = gbal_c[0] | gbal_c[1] | gbal_c[2];
    const int entry_grant = nb0 + grants + __popc(gbal & lanemask_lt());
    // the entry of my new page: the last grant of my class at or before me
    const unsigned mine = gbal_c[c] & (lanemask_lt() | (1u << lane));
    const int src = mine ? 31 - __clz(mine) : lane;
    const int entry_from = __shfl_sync(0xFFFFFFFFu, entry_grant, src);
    int entry = 0, slot = 0;
    uint32_t page = 0;
    uint32_t old_mask = 1;
    if (valid) {
      if (is_pop) {
        int32_t ts = C.free_slots[((int64_t)s * 3 + c) * cap + (F[c] - 1 - k)];
        entry = ts >> 4;
        slot = ts & 15;
        // through L2: an earlier batch of this call may have set bits of this
        // entry with atomics, which L1 does not see
        const uint64_t ent = __ldcg(&table[entry]);
        page = entry_page(ent);
        old_mask = entry_mask(ent);
      } else {
        entry = mine ? entry_from : last_entry[c];
        slot = slot_new;
        page = (uint32_t)(page_base[c] + j);
      }
    }
    // live-list candidates: granted entries, and reused entries with no live
    // token (an entry is in the live list exactly while its mask is non-zero)
    const bool cand = valid && (is_grant || (is_pop && old_mask == 0));
    const int key = cand ? entry : -1 - lane;
    const unsigned grp = __match_any_sync(0xFFFFFFFFu, key);
    const bool adder = cand && (__ffs(grp) - 1) == lane;
    const unsigned abal = __ballot_sync(0xFFFFFFFFu, adder);
    if (adder) {
      int at = nlive + __popc(abal & lanemask_lt());
      llist[at] = make_live_desc(page, c, entry);
      lidx[entry] = at;
    }
    nlive += __popc(abal);
    if (valid) {
      const int64_t sp = (int64_t)page * kPage;
      if (is_grant) {
        int used = min(kPage, cnt_in[c] - F[c] - (j << 4));
        uint32_t mask = (used >= 16) ? 0xFFFFu : ((1u << used) - 1u);
        table[entry] = make_entry(page, c, mask);
        for (int sl = used; sl < kPage; ++sl) C.slot_pos[c][sp + sl] = -1;
      } else if (is_pop) {
        atomicOr(reinterpret_cast<unsigned long long*>(&table[entry]),
                 (unsigned long long)(1ull << (48 + slot)));
      }
      C.slot_pos[c][sp + slot] = pos[i];
      C.fifo[((int64_t)s * 3 + c) * cap + ((int64_t)tail[c] + k) % cap] = entry * kPage + slot;
      tok_slot[i] = (int32_t)(sp + slot);
    }
#pragma unroll
    for (int cc = 0; cc < 3; ++cc) {
      rank[cc] += __popc(bal[cc]);
      if (gbal_c[cc]) last_entry[cc] = __shfl_sync(0xFFFFFFFFu, entry_grant, 31 - __clz(gbal_c[cc]));
    }
    grants += __popc(gbal);
    __syncwarp();
  }
  // final free stacks, FIFO tails and counters
#pragma unroll
  for (int cc = 0; cc < 3; ++cc) {
    int32_t* stack = C.free_slots + ((int64_t)s * 3 + cc) * cap;
    int cnt = cnt_in[cc];
    int top;
    if (cnt <= F[cc]) {
      top = F[cc] - cnt;
    } else {
      int over = cnt - F[cc];
      int u_last = over - (((over - 1) >> 4) << 4);  // slots used in the last new page
      top = kPage - u_last;
      for (int x = lane; x < top; x += 32) stack[x] = last_entry[cc] * kPage + (kPage - 1 - x);
    }
    if (lane == 0) {
      C.free_top[s * 3 + cc] = top;
      C.fifo_tail[s * 3 + cc] = tail[cc] + cnt;
    }
  }
  if (lane == 0) {
    C.num_blocks[s] = nb0 + grants;
    C.num_live[s] = nlive;
    if (st) C.live_count[s] = st[8] + len;
    else C.live_count[s] += len;
  }
}

__global__ void __launch_bounds__(kAssignThreads, 1)
    append_assign_kernel(CacheView C, int32_t n, const int32_t* __restrict__ seq,
                         const int32_t* __restrict__ pos, const uint8_t* __restrict__ tag,
                         AppendWorkspace ws, const int32_t* __restrict__ budget) {
  extern __shared__ uint32_t seen[];  // max_seqs bits
  __shared__ int s_err;
  __shared__ int s_blocks_bad;
  __shared__ int sh[40];
  __shared__ int s_nruns;
  __shared__ int s_total[3];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int max_seqs = C.L.max_seqs, nb_max = C.L.max_blocks_per_seq;

  if (tid == 0) {
    s_err = (*C.status != 0) ? -1 : 0;
    s_blocks_bad = 0;
    *ws.ok = 0;
  }
  for (int i = tid; i < (max_seqs + 31) / 32; i += kAssignThreads) seen[i] = 0;
  __syncthreads();
  if (s_err != 0) return;

  // ---- phase 1: validate, mark run starts --------------------------------
  int nruns_base = 0;
  for (int base = 0; base < n; base += kAssignThreads) {
    int i = base + tid;
    int start = 0;
    if (i < n) {
      int s = seq[i], c = tag[i], p = pos[i];
      bool bad = s < 0 || s >= max_seqs || c > 2 || p < 0;
      start = (i == 0) || seq[i - 1] != s;
      if (!bad && !start && p <= pos[i - 1]) bad = true;
      if (!bad && start && budget != nullptr && budget[i] < 0) bad = true;   // the evict that follows
      if (!bad && start) {
        uint32_t old = atomicOr(&seen[s >> 5], 1u << (s & 31));
        if (old & (1u << (s & 31))) bad = true;  // a sequence in two runs
      }
      if (bad) s_err = THINKV_ERR_INVALID;
    }
    int total;
    int excl = block_exclusive_scan(start, sh, &total);
    if (start) ws.runs[nruns_base + excl].start = i;
    nruns_base += total;
  }
  if (tid == 0) s_nruns = nruns_base;
  __syncthreads();
  if (s_err != 0) {
    if (tid == 0) set_status(C.status, s_err);
    return;
  }
  const int R = s_nruns;

  // ---- phase 2: per-run demand (warp per run) ------------------------------
  for (int r = warp; r < R; r += kAssignWarps) {
    int start = ws.runs[r].start;
    int end = (r + 1 < R) ? ws.runs[r + 1].start : n;
    int s = seq[start];
    int cnt[3] = {0, 0, 0};
    for (int i = start + lane; i - lane < end; i += 32) {
      int c = (i < end) ? tag[i] : -1;
#pragma unroll
      for (int cc = 0; cc < 3; ++cc) cnt[cc] += __popc(__ballot_sync(0xFFFFFFFFu, c == cc));
    }
    if (lane == 0) {
      int gs = 0;
      RunInfo& ri = ws.runs[r];
      ri.len = end - start;
      ri.seq = s;
#pragma unroll
      for (int cc = 0; cc < 3; ++cc) {
        int need = cnt[cc] - C.free_top[s * 3 + cc];
        int g = need > 0 ? (need + kPage - 1) / kPage : 0;
        ri.cnt[cc] = cnt[cc];
        ri.grants[cc] = g;
        gs += g;
      }
      if ((int64_t)C.num_blocks[s] + gs > nb_max) s_blocks_bad = 1;
    }
  }
  __syncthreads();

  // ---- phase 3: page grants in call order (exclusive scan per class) -------
  for (int cc = 0; cc < 3; ++cc) {
    int carry = 0;
    for (int base = 0; base < R; base += kAssignThreads) {
      int r = base + tid;
      int g = r < R ? ws.runs[r].grants[cc] : 0;
      int total;
      int excl = block_exclusive_scan(g, sh, &total);
      if (r < R) ws.runs[r].page_base[cc] = C.page_bump[cc] + carry + excl;
      carry += total;
    }
    if (tid == 0) s_total[cc] = carry;
  }
  __syncthreads();
  if (tid == 0) {
    int err = 0;
    if (s_blocks_bad) err = THINKV_ERR_OUT_OF_BLOCKS;
    for (int cc = 0; cc < 3; ++cc)
      if ((int64_t)C.page_bump[cc] + s_total[cc] > C.L.pool_pages[cc]) err = THINKV_ERR_OUT_OF_PAGES;
    s_err = err;
    if (err) set_status(C.status, err);
  }
  __syncthreads();
  if (s_err != 0) return;

  // ---- phase 4: slot assignment, warp per run ------------------------------
  for (int r = warp; r < R; r += kAssignWarps) {
    const RunInfo ri = ws.runs[r];
    assign_run(C, ri.seq, ri.start, ri.len, ri.cnt, ri.page_base, pos, tag, ws.tok_slot);
  }
  __syncthreads();
  if (tid == 0) {
    for (int cc = 0; cc < 3; ++cc) C.page_bump[cc] += s_total[cc];
    __threadfence();
    *ws.ok = 1;
  }
}

// ---------------------------------------------------------------------------
// quantise + scatter: one warp per (token, kv-head, K|V)
// ---------------------------------------------------------------------------
template <int D>
struct ScatterSmem {
  uint16_t code[D];  // codes (b <= 8) or raw fp16 bits (b == 16)
};

// This lane's D/32 channels of one K or V row (fp16 bits).
template <int D>
struct RowVals {
  uint16_t raw[D / 32];
};

template <int D>
__device__ inline RowVals<D> load_row(const uint16_t* __restrict__ x) {
  const int lane = threadIdx.x & 31;
  RowVals<D> r;
  if constexpr (D == 128) {
    uint2 v = *reinterpret_cast<const uint2*>(x + lane * 4);
    r.raw[0] = v.x & 0xFFFF; r.raw[1] = v.x >> 16; r.raw[2] = v.y & 0xFFFF; r.raw[3] = v.y >> 16;
  } else {
    uint32_t v = *reinterpret_cast<const uint32_t*>(x + lane * 2);
    r.raw[0] = v & 0xFFFF; r.raw[1] = v >> 16;
  }
  return r;
}

// Quantises one K or V row of one kv-head (values held by the warp, D/32
// channels per lane) at bit width B (class c) and writes its codes and params
// into slot pool_slot & 15 of page pool_slot >> 4's page-head block.
// F = 0: integer asymmetric codes.  F = 1: the float formats -- FP8 E4M3 (B =
// 8) and FP4 E2M1 (B = 4) with scale = fp16 rounded up of amax / (largest
// finite value) and zero 0; ternary (B = 2) with scale = fp16 rounded up of
// amax, code = clamp(rint_even(x / scale), -1, 1) + 1 and zero = -scale.
template <int D, int G, int B, int F>
__device__ void scatter_unit_b(const CacheView& C, int c, uint32_t pool_slot, int h, int kv,
                               const RowVals<D>& vals, uint16_t* code_sm) {
  constexpr int PER = D / 32;          // channels per lane
  constexpr int LPG = G / PER;         // lanes per group
  constexpr int NG = D / G;
  const int lane = threadIdx.x & 31;
  const uint32_t page = pool_slot >> 4, slot = pool_slot & 15;
  const int64_t phb = page_head_bytes(D, G, B);
  uint8_t* blk = C.pool[c] + ((int64_t)page * C.L.num_kv_heads + h) * phb;
  const uint16_t* raw = vals.raw;
  if constexpr (B == 16) {
#pragma unroll
    for (int e = 0; e < PER; ++e) code_sm[lane * PER + e] = raw[e];
  } else if constexpr (F == 1) {
    float xf[PER], amax = 0.f;
#pragma unroll
    for (int e = 0; e < PER; ++e) {
      xf[e] = __half2float(__ushort_as_half(raw[e]));
      amax = fmaxf(amax, fabsf(xf[e]));
    }
#pragma unroll
    for (int o = 1; o < LPG; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
    constexpr float top = B == 8 ? 448.f : (B == 4 ? 6.f : 1.f);
    const __half sh = __float2half_ru(__fdiv_rn(amax, top));
    const float sf = __half2float(sh);
#pragma unroll
    for (int e = 0; e < PER; ++e) {
      uint32_t cq;
      if constexpr (B == 2) {
        float r = sf == 0.f ? 0.f : rintf(__fdiv_rn(xf[e], sf));
        r = fminf(fmaxf(r, -1.f), 1.f);
        cq = (uint32_t)((int)r + 1);
      } else {
        const float t = sf == 0.f ? 0.f : __fdiv_rn(xf[e], sf);
        cq = B == 8 ? e4m3_code(t) : e2m1_code(t);
      }
      code_sm[lane * PER + e] = (uint16_t)cq;
    }
    const int grp = (lane * PER) / G;
    if ((lane % LPG) == 0) {
      uint16_t* prm = reinterpret_cast<uint16_t*>(blk + 4LL * D * B + (kv ? 64LL * NG : 0));
      const uint16_t zb = B == 2 ? (uint16_t)(__half_as_ushort(sh) ^ 0x8000u) : (uint16_t)0;
      const uint32_t pair = (uint32_t)__half_as_ushort(sh) | ((uint32_t)zb << 16);
      *reinterpret_cast<uint32_t*>(prm + (grp * 16 + slot) * 2) = pair;
    }
  } else {
    float xf[PER], mn = INFINITY, mx = -INFINITY;
#pragma unroll
    for (int e = 0; e < PER; ++e) {
      xf[e] = __half2float(__ushort_as_half(raw[e]));
      mn = fminf(mn, xf[e]);
      mx = fmaxf(mx, xf[e]);
    }
#pragma unroll
    for (int o = 1; o < LPG; o <<= 1) {
      mn = fminf(mn, __shfl_xor_sync(0xFFFFFFFFu, mn, o));
      mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
    }
    const __half zh = __float2half_rd(mn);
    const float zf = __half2float(zh);
    constexpr float levels = (float)((1 << B) - 1);
    const float s32 = __fdiv_rn(__fsub_rn(mx, zf), levels);
    const __half sh = __float2half_ru(s32);
    const float sf = __half2float(sh);
#pragma unroll
    for (int e = 0; e < PER; ++e) {
      int cq = 0;
      if (sf != 0.0f) {
        float t = __fdiv_rn(__fsub_rn(xf[e], zf), sf);
        float r = rintf(t);
        r = fminf(fmaxf(r, 0.0f), levels);
        cq = (int)r;
      }
      code_sm[lane * PER + e] = (uint16_t)cq;
    }
    const int grp = (lane * PER) / G;
    if ((lane % LPG) == 0) {
      uint16_t* prm = reinterpret_cast<uint16_t*>(blk + 4LL * D * B + (kv ? 64LL * NG : 0));
      uint32_t pair = (uint32_t)__half_as_ushort(sh) | ((uint32_t)__half_as_ushort(zh) << 16);
      *reinterpret_cast<uint32_t*>(prm + (grp * 16 + slot) * 2) = pair;
    }
  }
  __syncwarp();

  constexpr int lane_bytes = D * B / 16;
  uint8_t* region = blk + (kv ? 2LL * D * B : 0);
  if (kv == 0) {
    // K: pieces (layout lane 4*(slot%8)+t, group gr, r = slot/8) of G/4 channels
    constexpr int pb = G * B / 32;                 // piece bytes (>= 2)
    if (lane < 4 * NG) {
      const int t = lane & 3, gr = lane >> 2;
      const int l = 4 * (slot & 7) + t, r = slot >> 3;
      const uint16_t* src = code_sm + gr * G + t * (G / 4);
      if constexpr (B == 16) {
        // raw fp16: the piece is G/4 channels in natural order
        const int o = (gr * 2 + r) * pb;
#pragma unroll
        for (int e = 0; e < G / 4; e += 2)
          *reinterpret_cast<uint32_t*>(region + lane_off(l, o + 2 * e, lane_bytes)) =
              (uint32_t)src[e] | ((uint32_t)src[e + 1] << 16);
      } else {
        constexpr int m = (32 / B) < (G / 4) ? (32 / B) : (G / 4);   // channels per word
        uint32_t words[4] = {0, 0, 0, 0};
#pragma unroll
        for (int e = 0; e < G / 4; ++e) {
          const uint32_t v = src[e];
          const int wi = e / m, el = e % m;
          const int p = (el & 1) ? (m / 2 + el / 2) : (el / 2);
          words[wi] |= v << (p * B);
        }
        uint8_t* dst = region + lane_off(l, (gr * 2 + r) * pb, lane_bytes);   // pb <= chunk
        if constexpr (pb == 2) *reinterpret_cast<uint16_t*>(dst) = (uint16_t)words[0];
        else if constexpr (pb == 4) *reinterpret_cast<uint32_t*>(dst) = words[0];
        else if constexpr (pb == 8) *reinterpret_cast<uint2*>(dst) = make_uint2(words[0], words[1]);
        else *reinterpret_cast<uint4*>(dst) = make_uint4(words[0], words[1], words[2], words[3]);
      }
    }
  } else {
    // V: half-words (lane 4*g + t, P, q, half) holding 16/B codes each
    const int t = (slot & 7) >> 1, P = slot >> 3, half = slot & 1;
    constexpr int Q = D * B / 128;                 // chunks per P
    constexpr int per = 16 / B;                    // codes per half-word
#pragma unroll
    for (int u0 = 0; u0 < 8 * Q; u0 += 32) {
      const int u = u0 + lane;
      if (u < 8 * Q) {
        const int g = u / Q, q = u % Q;
        uint32_t hw = 0;
#pragma unroll
        for (int k = 0; k < per; ++k) {
          const int e = q * per + k;
          const int ch = 16 * (e >> 1) + g + 8 * (e & 1);
          hw |= (uint32_t)code_sm[ch] << (B * k);
        }
        const int l = 4 * g + t;
        uint8_t* dst = region + lane_off(l, (P * Q + q) * 4 + 2 * half, lane_bytes);
        *reinterpret_cast<uint16_t*>(dst) = (uint16_t)hw;
      }
    }
  }
  __syncwarp();
}

template <int D, int G>
__device__ inline void scatter_unit(const CacheView& C, int c, uint32_t pool_slot, int h, int kv,
                                    const RowVals<D>& vals, uint16_t* code_sm) {
  switch (C.L.bits[c] + (C.L.fmt[c] == 1 ? 256 : 0)) {
    case 8: scatter_unit_b<D, G, 8, 0>(C, c, pool_slot, h, kv, vals, code_sm); break;
    case 4: scatter_unit_b<D, G, 4, 0>(C, c, pool_slot, h, kv, vals, code_sm); break;
    case 2: scatter_unit_b<D, G, 2, 0>(C, c, pool_slot, h, kv, vals, code_sm); break;
    case 256 + 8: scatter_unit_b<D, G, 8, 1>(C, c, pool_slot, h, kv, vals, code_sm); break;
    case 256 + 4: scatter_unit_b<D, G, 4, 1>(C, c, pool_slot, h, kv, vals, code_sm); break;
    case 256 + 2: scatter_unit_b<D, G, 2, 1>(C, c, pool_slot, h, kv, vals, code_sm); break;
    default: scatter_unit_b<D, G, 16, 0>(C, c, pool_slot, h, kv, vals, code_sm); break;
  }
}

template <int D, int G>
__global__ void __launch_bounds__(256)
    append_scatter_kernel(CacheView C, int32_t n, const uint8_t* __restrict__ tag,
                          const uint16_t* __restrict__ k, const uint16_t* __restrict__ v,
                          AppendWorkspace ws) {
  __shared__ ScatterSmem<D> sm[8];
  if (*ws.ok == 0) return;
  const int warp = threadIdx.x >> 5;
  const int H = C.L.num_kv_heads;
  const int64_t units = (int64_t)n * H * 2;
  for (int64_t u = (int64_t)blockIdx.x * 8 + warp; u < units; u += (int64_t)gridDim.x * 8) {
    const int kv = (int)(u & 1);
    const int64_t th = u >> 1;
    const int h = (int)(th % H);
    const int64_t i = th / H;
    const int c = tag[i];
    const uint16_t* x = (kv ? v : k) + (i * H + h) * D;
    scatter_unit<D, G>(C, c, (uint32_t)ws.tok_slot[i], h, kv, load_row<D>(x), sm[warp].code);
  }
}


// ---------------------------------------------------------------------------
// small calls (n <= kSmallAppend tokens, e.g. one token per sequence of a
// decode step): one launch.  Every CTA validates the whole call and builds
// the run table and the page grants in shared memory -- the same result in
// every CTA, so no grid-wide barrier is needed.  CTA r then assigns run r's
// slots (warp 0) and quantises and stores run r's tokens (all warps).  The
// page-pool counters are advanced by the last CTA to finish (an arrival
// counter in the workspace): every CTA reads them before it arrives.
// ---------------------------------------------------------------------------
constexpr int kSmallThreads = 256;
constexpr int kSmallWarps = kSmallThreads / 32;
constexpr int kSmallPer = kSmallAppend / kSmallThreads;   // tokens per thread, contiguous

// Block-wide exclusive scan over kSmallThreads threads (sh: >= kSmallWarps + 1 ints).
__device__ int small_exclusive_scan(int v, int* sh, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xFFFFFFFFu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sh[warp] = x;
  __syncthreads();
  int base = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < kSmallWarps; ++w) {
    const int t = sh[w];
    base += (w < warp) ? t : 0;
    tot += t;
  }
  __syncthreads();
  *total = tot;
  return base + x - v;
}

// Block-wide sum of NV values per thread (sh: >= NV * kSmallWarps ints).
template <int NV>
__device__ void small_block_sum(int (&v)[NV], int* sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int j = 0; j < NV; ++j) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v[j] += __shfl_xor_sync(0xFFFFFFFFu, v[j], o);
    if (lane == 0) sh[j * kSmallWarps + warp] = v[j];
  }
  __syncthreads();
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    int t = 0;
#pragma unroll
    for (int w = 0; w < kSmallWarps; ++w) t += sh[j * kSmallWarps + w];
    v[j] = t;
  }
  __syncthreads();
}

template <int D, int G>
__global__ void __launch_bounds__(kSmallThreads)
    append_small_kernel(CacheView C, int32_t n, const int32_t* __restrict__ seq,
                        const int32_t* __restrict__ pos, const uint8_t* __restrict__ tag,
                        const uint16_t* __restrict__ k, const uint16_t* __restrict__ v,
                        uint32_t* arrive, const int32_t* __restrict__ budget, uint32_t order) {
  constexpr int NST = 9;                          // counters per run (see assign_run)
  extern __shared__ uint32_t seen[];              // max_seqs bits
  __shared__ int r_cnt[kSmallAppend * 3];         // per run: tokens of each class
  __shared__ int r_st[kSmallAppend * NST];        // per run: its sequence's counters
  __shared__ int r_start[kSmallAppend + 1];       // per run: first token (r_start[R] = n)
  __shared__ int r_seq[kSmallAppend];
  __shared__ int32_t tok_slot[kSmallAppend];      // pool slots of this CTA's run
  __shared__ ScatterSmem<D> sm[kSmallWarps];
  __shared__ int sh[8 * kSmallWarps];
  __shared__ int s_err, s_base[3], s_total[3], s_bump[3], s_blocks_bad;
  const int tid = threadIdx.x, warp = tid >> 5;
  const int max_seqs = C.L.max_seqs, nb_max = C.L.max_blocks_per_seq, H = C.L.num_kv_heads;
  const int b = blockIdx.x;                       // the run this CTA owns (if any)
  // the next kernel may be scheduled at once -- unless this launch also
  // evicts: then its CTAs live long enough that an early decode grid would
  // find SMs short of registers, so each CTA signals once its work is done
  if (budget == nullptr) pdl_launch_dependents();

  // ---- the call's own inputs (before the previous kernel has finished) ----
  // speculative prefetch: with one token per run (a decode step), run b is
  // token b; its first K/V rows are loaded while the call is validated
  RowVals<D> pre, pre2;
  const bool pre_ok = b < n && warp < 2 * H;
  const bool pre2_ok = b < n && warp + kSmallWarps < 2 * H;
  if (pre_ok) {
    const int h = warp >> 1, kv = warp & 1;
    pre = load_row<D>((kv ? v : k) + ((int64_t)b * H + h) * D);
  }
  if (pre2_ok) {                                  // the warp's second unit of token b
    const int u2 = warp + kSmallWarps, h = u2 >> 1, kv = u2 & 1;
    pre2 = load_row<D>((kv ? v : k) + ((int64_t)b * H + h) * D);
  }
  const int pre_tag = b < n ? tag[b] : 0;
  const int x0 = tid * kSmallPer;
  int s_[kSmallPer], c_[kSmallPer], p_[kSmallPer], sp_[kSmallPer], pp_[kSmallPer];
#pragma unroll
  for (int e = 0; e < kSmallPer; ++e) {
    const int x = x0 + e;
    s_[e] = -1; c_[e] = 0; p_[e] = 0; sp_[e] = -1; pp_[e] = 0;
    if (x < n) {
      s_[e] = seq[x]; c_[e] = tag[x]; p_[e] = pos[x];
      if (x > 0) { sp_[e] = seq[x - 1]; pp_[e] = pos[x - 1]; }
    }
  }
  for (int i = tid; i < (max_seqs + 31) / 32; i += kSmallThreads) seen[i] = 0;
  for (int i = tid; i < kSmallAppend * 3; i += kSmallThreads) r_cnt[i] = 0;
  if (tid == 0) s_err = 0;
  __syncthreads();

  // ---- validate; run starts ----
  int nstart = 0, first_s = -1;
  bool bad = false;
#pragma unroll
  for (int e = 0; e < kSmallPer; ++e) {
    const int x = x0 + e;
    if (x >= n) break;
    const int s = s_[e], c = c_[e], p = p_[e];
    const bool start = (x == 0) || sp_[e] != s;
    bool bx = s < 0 || s >= max_seqs || c > 2 || p < 0;
    if (!bx && !start && p <= pp_[e]) bx = true;
    if (!bx && start && budget != nullptr && budget[x] < 0) bx = true;   // the evict that follows
    if (!bx && start) {
      const uint32_t old = atomicOr(&seen[s >> 5], 1u << (s & 31));
      if (old & (1u << (s & 31))) bx = true;          // a sequence in two runs
    }
    if (start && nstart == 0 && !bx) first_s = s;
    bad |= bx;
    nstart += start;
  }
  if (bad) s_err = THINKV_ERR_INVALID;

  // ---- cache state: only once the previous kernel is done ----
  pdl_wait();
  int st0[NST];                                   // counters of the first run starting here
  if (first_s >= 0) {
    const int s = first_s;
#pragma unroll
    for (int c = 0; c < 3; ++c) {
      st0[c] = C.free_top[s * 3 + c];
      st0[3 + c] = C.fifo_tail[s * 3 + c];
    }
    st0[6] = C.num_blocks[s];
    st0[7] = C.num_live[s];
    st0[8] = C.live_count[s];
  }
  if (tid == 0) {
    if (*C.status != 0) s_err = -1;
    s_blocks_bad = 0;
#pragma unroll
    for (int c = 0; c < 3; ++c) s_bump[c] = C.page_bump[c];
  }
  int R;
  const int rbase = small_exclusive_scan(nstart, sh, &R);   // (its barriers publish s_err)
  if (s_err != 0) {
    if (b == 0 && tid == 0 && s_err > 0) set_status(C.status, s_err);
    return;
  }
  {
    int r = rbase - 1;                              // run of the token before my first
    bool first_start = true;
#pragma unroll
    for (int e = 0; e < kSmallPer; ++e) {
      const int x = x0 + e;
      if (x >= n) break;
      const bool start = (x == 0) || sp_[e] != s_[e];
      if (start) {
        ++r;
        r_start[r] = x;
        r_seq[r] = s_[e];
        const int s = s_[e];
#pragma unroll
        for (int c = 0; c < 3; ++c) {
          r_st[r * NST + c] = first_start ? st0[c] : C.free_top[s * 3 + c];
          r_st[r * NST + 3 + c] = first_start ? st0[3 + c] : C.fifo_tail[s * 3 + c];
        }
        r_st[r * NST + 6] = first_start ? st0[6] : C.num_blocks[s];
        r_st[r * NST + 7] = first_start ? st0[7] : C.num_live[s];
        r_st[r * NST + 8] = first_start ? st0[8] : C.live_count[s];
        first_start = false;
      }
      atomicAdd(&r_cnt[r * 3 + c_[e]], 1);
    }
  }
  if (tid == 0) r_start[R] = n;
  __syncthreads();

  // ---- page grants in call order: my run's bases and the call's totals ----
  {
    int acc[6] = {0, 0, 0, 0, 0, 0};              // grants of runs before b (3), all runs (3)
    for (int r = tid; r < R; r += kSmallThreads) {
      int gs = 0;
#pragma unroll
      for (int c = 0; c < 3; ++c) {
        const int need = r_cnt[r * 3 + c] - r_st[r * NST + c];
        const int g = need > 0 ? (need + kPage - 1) / kPage : 0;
        acc[c] += (r < b) ? g : 0;
        acc[3 + c] += g;
        gs += g;
      }
      if ((int64_t)r_st[r * NST + 6] + gs > nb_max) s_blocks_bad = 1;
    }
    small_block_sum<6>(acc, sh);
    if (tid == 0) {
#pragma unroll
      for (int c = 0; c < 3; ++c) {
        s_base[c] = s_bump[c] + acc[c];
        s_total[c] = acc[3 + c];
      }
      int err = 0;
      if (s_blocks_bad) err = THINKV_ERR_OUT_OF_BLOCKS;
#pragma unroll
      for (int c = 0; c < 3; ++c)
        if ((int64_t)s_bump[c] + acc[3 + c] > C.L.pool_pages[c]) err = THINKV_ERR_OUT_OF_PAGES;
      s_err = err;
    }
    __syncthreads();
    if (s_err != 0) {
      if (b == 0 && tid == 0) set_status(C.status, s_err);
      return;
    }
  }

  // ---- run b: slots (warp 0), then quantise + store its tokens (all warps) ----
  if (b < R) {
    const int start = r_start[b], len = r_start[b + 1] - start, s = r_seq[b];
    if (warp == 0) {
      const int cnt[3] = {r_cnt[b * 3 + 0], r_cnt[b * 3 + 1], r_cnt[b * 3 + 2]};
      const int base[3] = {s_base[0], s_base[1], s_base[2]};
      assign_run(C, s, start, len, cnt, base, pos, tag, tok_slot - start, r_st + b * NST);
    }
    __syncthreads();
    // append + evict: warp 0 then takes the sequence down to its budget (its
    // counters are final once the barrier has passed; the other warps store
    // the run's codes meanwhile, into slots the evict does not read)
    if (budget != nullptr && warp == 0) evict_seq(C, s, budget[start], order, false);
    const int64_t units = (int64_t)len * H * 2;
    for (int64_t u = warp; u < units; u += kSmallWarps) {
      const int kv = (int)(u & 1);
      const int64_t th = u >> 1;
      const int h = (int)(th % H);
      const int i = start + (int)(th / H);
      const bool own = start == b;                  // token b opens run b: prefetched
      const RowVals<D> vals = (u == warp && pre_ok && own)                 ? pre
                              : (u == warp + kSmallWarps && pre2_ok && own) ? pre2
                              : load_row<D>((kv ? v : k) + ((int64_t)i * H + h) * D);
      scatter_unit<D, G>(C, (own && i == b) ? pre_tag : tag[i], (uint32_t)tok_slot[i - start], h,
                         kv, vals, sm[warp].code);
    }
  }

  // ---- the last CTA to finish advances the page-pool counters ----
  __syncthreads();
  if (budget != nullptr) pdl_launch_dependents();
  if (tid == 0) {
    __threadfence();
    const uint32_t old = atomicAdd(arrive, 1u);
    if (old == gridDim.x - 1) {
#pragma unroll
      for (int c = 0; c < 3; ++c) C.page_bump[c] = s_bump[c] + s_total[c];
      *arrive = 0u;
    }
  }
}
}  // namespace

size_t append_workspace_bytes(int32_t n) {
  size_t bytes = 256;                                   // ok flag
  bytes += ((size_t)n * sizeof(int32_t) + 255) / 256 * 256;
  bytes += ((size_t)(n > 0 ? n : 1) * sizeof(RunInfo) + 255) / 256 * 256;
  return bytes;
}

AppendWorkspace carve_append_workspace(void* ws, int32_t n) {
  AppendWorkspace w;
  uint8_t* p = static_cast<uint8_t*>(ws);
  w.arrive = reinterpret_cast<uint32_t*>(p);        // bytes [0, 4): left zero by every call
  w.ok = reinterpret_cast<int32_t*>(p + 128);
  p += 256;
  w.tok_slot = reinterpret_cast<int32_t*>(p);
  p += ((size_t)n * sizeof(int32_t) + 255) / 256 * 256;
  w.runs = reinterpret_cast<RunInfo*>(p);
  return w;
}

cudaError_t launch_append(const CacheView& C, int32_t n, const int32_t* seq, const int32_t* pos,
                          const uint8_t* tag, const uint16_t* k, const uint16_t* v,
                          const AppendWorkspace& ws, cudaStream_t stream, int num_sms,
                          const int32_t* budget, const uint8_t* order) {
  const size_t seen_bytes = (size_t)((C.L.max_seqs + 31) / 32) * 4;
  const int D = C.L.head_dim, G = C.L.group_size;
  const uint32_t packed =
      order ? ((uint32_t)order[0] | ((uint32_t)order[1] << 8) | ((uint32_t)order[2] << 16)) : 0u;
  if (n <= kSmallAppend) {
    auto kern = (D == 128 && G == 64)   ? append_small_kernel<128, 64>
                : (D == 128 && G == 32) ? append_small_kernel<128, 32>
                : (D == 64 && G == 64)  ? append_small_kernel<64, 64>
                                        : append_small_kernel<64, 32>;
    return launch_pdl(kern, dim3(n), dim3(kSmallThreads), seen_bytes, stream, C, n, seq, pos, tag,
                      k, v, ws.arrive, budget, packed);
  }
  append_assign_kernel<<<1, kAssignThreads, seen_bytes, stream>>>(C, n, seq, pos, tag, ws, budget);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  const int64_t units = (int64_t)n * C.L.num_kv_heads * 2;
  int64_t blocks = (units + 7) / 8;
  const int64_t cap = (int64_t)num_sms * 16;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  if (D == 128 && G == 64) append_scatter_kernel<128, 64><<<(int)blocks, 256, 0, stream>>>(C, n, tag, k, v, ws);
  else if (D == 128 && G == 32) append_scatter_kernel<128, 32><<<(int)blocks, 256, 0, stream>>>(C, n, tag, k, v, ws);
  else if (D == 64 && G == 64) append_scatter_kernel<64, 64><<<(int)blocks, 256, 0, stream>>>(C, n, tag, k, v, ws);
  else append_scatter_kernel<64, 32><<<(int)blocks, 256, 0, stream>>>(C, n, tag, k, v, ws);
  err = cudaGetLastError();
  if (err != cudaSuccess || budget == nullptr) return err;
  // append + evict on a large call: each run's sequence to its budget
  return launch_evict_runs(C, n, seq, budget, order, stream);
}

}  // namespace thinkv
