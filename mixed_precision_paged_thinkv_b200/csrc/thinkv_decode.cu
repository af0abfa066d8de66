// thinkv_decode.cu -- decode attention over mixed-precision, slot-reusing pages.
//
// "ThinKV: Thought-Adaptive KV Cache Compression for Efficient Reasoning
// Models": the arXiv abstract's kernel "that extends PagedAttention" to read a
// cache whose tokens carry per-thought-type precision (explainer, Methodologie,
// TBQ) and whose evicted slots are holes that are never compacted (explainer,
// "Implementation Systeme: Pensee Continue (CT)").  The pages print no kernel
// design; this one is written for sm_100a:
//
//   split kernel (stream-K): the live page-heads of all decoded sequences form
//   one ordered list of units (sequence, kv-head, live page); every warp of the
//   grid takes an equal contiguous share, so work is balanced by live pages no
//   matter how lengths and budgets vary.  Per warp, lane 0 streams page-head
//   blocks (K codes, V codes, params: one contiguous block per page and head)
//   into a shared-memory ring with cp.async.bulk (TMA) + mbarriers; the warp
//   unpacks codes straight into mma.sync m16n8k16 operands (fp16 magic-number
//   conversion, codes centred by 2^(b-1) so products stay exact), computes
//   q.k for the whole GQA group at once (tokens x heads), applies the per-group
//   scale/zero in fp32, runs the online softmax, transposes p through a small
//   shared buffer and accumulates p*scale (fp16, exponent-shifted) times the V
//   codes on the tensor cores, with the zero terms summed in fp32.  Each warp
//   writes one partial (m, l, o, top-k logits) per (sequence, kv-head) segment
//   it touched and counts itself in on the segment's arrival counter; the
//   last warp to arrive merges the segment's partials with the log-sum-exp
//   rule and writes fp16 O and the top-k mass -- one launch per decode.
#include <cuda_fp16.h>
#include <stdint.h>

#include "thinkv_common.cuh"
#include "thinkv_internal.h"

namespace thinkv {

namespace {

constexpr int kDecWarps = 4;
constexpr int kDecThreads = kDecWarps * 32;
constexpr int kDecMinBlocks = 3;                       // CTAs per SM the kernel is built for
constexpr int kDecRegs = 65536 / (kDecThreads * kDecMinBlocks) / 8 * 8;  // register cap (168)
constexpr int kPbufStride = 12;                 // floats per row of the p transpose buffer
// per-warp scratch: during pages, the p transpose (16 x 12 floats) and the
// segment's Q fragments (lane-contiguous, up to 2 KB); during a merge, which
// runs between two segments, the (m, l) table of the pieces (32 x 8 float2 +
// 16 floats) overlays both
constexpr int kPtBytes = 16 * kPbufStride * 4;          // 768
constexpr int kQfragOff = kPtBytes;
constexpr int kQfragBytes = 2048;                       // (D / 16) k-steps x 32 lanes x 8 B
constexpr int kPbufBytes = kPtBytes + kQfragBytes;      // >= 2 * 32 * 8 * 4 + 16 * 4
constexpr int kSigmaInit = 1 << 20;
constexpr int kCandCap = 128;                   // top-k candidate slots per head
constexpr int kTopkHdrBytes = 64;               // per-head counts and thresholds

struct DecodeParams {
  const uint8_t* pool[3];
  int32_t phb[3];
  int32_t bits[3];
  const uint64_t* table;
  const uint64_t* live_list;
  const int32_t* num_live;
  int32_t max_blocks, max_seqs;
  int32_t Hkv, Hq, Gq;
  const int32_t* seq;
  int32_t n;
  const uint16_t* q;
  float scale_log2;
  float* part_o;   // [pieces][Gq][D]
  float* part_ml;  // [pieces][Gq][2]   (m in log2 units, l)
  float* part_topk;  // [pieces][Gq][topk] largest logits (log2 units), -inf padded
  uint32_t* ctr;     // [n * Hkv] arrival counters of the segments (zero between calls)
  const int32_t* live_count;
  uint16_t* out;     // [n][Hq][D]
  float* mass;       // [n][Hq] or null
  int32_t topk;
  int32_t* status;
  int32_t nstage, stage_bytes, warp_smem, plan_smem;
  int32_t q_off, q_bytes;  // Q rows of a segment ride with its first page: stage + q_off
};

__device__ inline float pow2i(int e) { return __int_as_float((127 + e) << 23); }

// ---------------------------------------------------------------------------
// top-k attention mass: candidate buffers
// ---------------------------------------------------------------------------
// Sorts 128 values held 4 per lane (element lane*4 + j) into descending order
// (bitonic network; exchanges across lanes use shuffles).
__device__ inline void bitonic128_desc(float (&v)[4]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int size = 2; size <= 128; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      if (stride >= 4) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int i = lane * 4 + j;
          const float o = __shfl_xor_sync(0xFFFFFFFFu, v[j], stride >> 2);
          const bool desc = (i & size) == 0, lower = (i & stride) == 0;
          v[j] = (lower == desc) ? fmaxf(v[j], o) : fminf(v[j], o);
        }
      } else {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          if (j & stride) continue;
          const int i = lane * 4 + j;
          const bool desc = (i & size) == 0;
          const float a = v[j], b = v[j | stride];
          v[j] = desc ? fmaxf(a, b) : fminf(a, b);
          v[j | stride] = desc ? fminf(a, b) : fmaxf(a, b);
        }
      }
    }
  }
}

struct TopkCtx {
  float* cand;    // [Gq][kCandCap]
  int* cnt;       // [Gq]
  float* theta;   // [Gq]  values <= theta cannot enter the top-k any more
  int topk;
};

// Keeps the topk largest candidates of head h and raises its threshold.
__device__ inline void cand_compact(const TopkCtx& tk, int h) {
  const int lane = threadIdx.x & 31;
  float* c = tk.cand + h * kCandCap;
  const int n = tk.cnt[h];
  float v[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) v[j] = (lane * 4 + j < n) ? c[lane * 4 + j] : -INFINITY;
  bitonic128_desc(v);
  __syncwarp();
  const int keep = min(n, tk.topk);
#pragma unroll
  for (int j = 0; j < 4; ++j)
    if (lane * 4 + j < keep) c[lane * 4 + j] = v[j];
  const int kl = tk.topk - 1;
  const float sel = (kl & 3) == 0 ? v[0] : (kl & 3) == 1 ? v[1] : (kl & 3) == 2 ? v[2] : v[3];
  const float kth = __shfl_sync(0xFFFFFFFFu, sel, kl >> 2);
  __syncwarp();
  if (lane == 0) {
    tk.cnt[h] = keep;
    if (n >= tk.topk) tk.theta[h] = kth;
  }
  __syncwarp();
}

// Merges the partials (m, l, o, top-k logits) of segment (i, h) into fp16 O
// and the top-k mass of its Gq query heads.  Run by the last warp to finish a
// piece of the segment.  Pieces are the non-empty warps from w0 on: with
// T <= W every unit has its own warp, otherwise all of w0..w1 hold units.
// Loads are issued lane-parallel or in independent batches (a loop of
// dependent loads would put one L2 round trip per piece on the kernel tail);
// partials are read through L2 (ld.global.cg).
__device__ inline int64_t piece_warp(int j, int64_t Us, int64_t w0, int64_t T, int64_t W) {
  return T <= W ? ((Us + j + 1) * W - 1) / T : w0 + j;
}

template <int D>
__device__ void merge_segment(const DecodeParams& p, int i, int h, int64_t Us,
                                           int64_t w0, int np, int64_t T, int64_t W,
                                           const TopkCtx& tk, float* scratch) {
  const int lane = threadIdx.x & 31;
  constexpr int QD = D / 4;                     // float4 quads per head row
  constexpr int CH = 32;                        // pieces per chunk (scratch: 2 * CH * 8 floats)
  const int Gq = p.Gq;
  const int64_t seg = (int64_t)i * p.Hkv + h;
  const int npair = Gq * QD;
  float2* ml = reinterpret_cast<float2*>(scratch);            // [CH][Gq] (m, l)
  float* Mh = scratch + 2 * CH * 8;                           // [Gq] running max
  float* Lh = Mh + 8;                                         // [Gq] row sums

  // ---- pass 1: M per head over all pieces ----
  if (lane < Gq) Mh[lane] = -INFINITY;
  __syncwarp();
  for (int jb = 0; jb < np; jb += CH) {
    const int cnt = min(CH, np - jb);
    for (int x = lane; x < cnt * Gq; x += 32) {
      const int j = x / Gq, r = x - j * Gq;
      const int64_t pc = (piece_warp(jb + j, Us, w0, T, W) + seg) * Gq + r;
      ml[x] = __ldcg(reinterpret_cast<const float2*>(p.part_ml + pc * 2));
    }
    __syncwarp();
    if (lane < Gq) {
      float mx = Mh[lane];
      for (int j = 0; j < cnt; ++j) mx = fmaxf(mx, ml[j * Gq + lane].x);
      Mh[lane] = mx;
    }
    __syncwarp();
  }
  // ---- pass 2: weights and row sums ----
  if (lane < Gq) Lh[lane] = 0.f;
  __syncwarp();
  // (head, quad) pairs of this lane: lane + 32 x; done in groups of PG pairs,
  // each over all pieces with BATCH pieces of independent loads in flight
  constexpr int PG = 4, BATCH = 4;
  const int npl = (npair + 31) / 32;
  for (int x0 = 0; x0 < npl; x0 += PG) {
    float4 acc[PG];
#pragma unroll
    for (int x = 0; x < PG; ++x) acc[x] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int jb = 0; jb < np; jb += CH) {
      const int cnt = min(CH, np - jb);
      if (np > CH || x0 > 0) {  // (m, l) of this chunk (a single chunk is still in scratch)
        for (int x = lane; x < cnt * Gq; x += 32) {
          const int j = x / Gq, r = x - j * Gq;
          const int64_t pc = (piece_warp(jb + j, Us, w0, T, W) + seg) * Gq + r;
          ml[x] = __ldcg(reinterpret_cast<const float2*>(p.part_ml + pc * 2));
        }
        __syncwarp();
      }
      for (int x = lane; x < cnt * Gq; x += 32) ml[x].x = exp2_approx(ml[x].x - Mh[x % Gq]);
      __syncwarp();
      if (x0 == 0 && lane < Gq) {
        float l = Lh[lane];
        for (int j = 0; j < cnt; ++j) l = fmaf(ml[j * Gq + lane].y, ml[j * Gq + lane].x, l);
        Lh[lane] = l;
      }
      for (int jj = 0; jj < cnt; jj += BATCH) {
        float4 v[BATCH][PG];
#pragma unroll
        for (int b = 0; b < BATCH; ++b) {
          if (jj + b < cnt) {
            const int64_t base = (piece_warp(jb + jj + b, Us, w0, T, W) + seg) * Gq;
#pragma unroll
            for (int x = 0; x < PG; ++x) {
              const int pr = lane + 32 * (x0 + x);
              if (pr < npair) {
                const int r = pr / QD, q = pr - r * QD;
                v[b][x] = __ldcg(reinterpret_cast<const float4*>(p.part_o + (base + r) * D) + q);
              }
            }
          }
        }
#pragma unroll
        for (int b = 0; b < BATCH; ++b) {
          if (jj + b < cnt) {
#pragma unroll
            for (int x = 0; x < PG; ++x) {
              const int pr = lane + 32 * (x0 + x);
              if (pr < npair) {
                const float fw = ml[(jj + b) * Gq + pr / QD].x;
                acc[x].x = fmaf(v[b][x].x, fw, acc[x].x);
                acc[x].y = fmaf(v[b][x].y, fw, acc[x].y);
                acc[x].z = fmaf(v[b][x].z, fw, acc[x].z);
                acc[x].w = fmaf(v[b][x].w, fw, acc[x].w);
              }
            }
          }
        }
      }
      __syncwarp();
    }
    // ---- fp16 output rows for this group of pairs ----
#pragma unroll
    for (int x = 0; x < PG; ++x) {
      const int pr = lane + 32 * (x0 + x);
      if (pr < npair) {
        const int r = pr / QD, q = pr - r * QD;
        const float inv = 1.f / Lh[r];
        const uint32_t lo = (uint32_t)__half_as_ushort(__float2half_rn(acc[x].x * inv)) |
                            ((uint32_t)__half_as_ushort(__float2half_rn(acc[x].y * inv)) << 16);
        const uint32_t hi = (uint32_t)__half_as_ushort(__float2half_rn(acc[x].z * inv)) |
                            ((uint32_t)__half_as_ushort(__float2half_rn(acc[x].w * inv)) << 16);
        const int64_t row = (int64_t)i * p.Hq + h * Gq + r;
        reinterpret_cast<uint2*>(p.out + row * D)[q] = make_uint2(lo, hi);
      }
    }
  }
  if (!p.mass) return;
  for (int r = 0; r < Gq; ++r) {
    const int64_t row = (int64_t)i * p.Hq + h * Gq + r;
    const float M = Mh[r];
    const float inv = 1.f / Lh[r];
    const int k = p.topk;
    if (p.live_count[p.seq[i]] <= k) {
      if (lane == 0) p.mass[row] = 1.f;
      continue;
    }
    // ---- top-k of the union of the pieces' top-k lists ----
    // Each list holds its piece's k largest logits (-inf padded), so the
    // union's k-th largest is >= theta = max over pieces of min(list): only
    // values >= theta can be in the top-k, and at least k of them exist.
    float v[4];
    bool done = false;
    const int staged = np * k;
    if (staged <= (Gq - 1) * kCandCap) {
      float* st = tk.cand;                                 // staging: np*k values
      float* sb = tk.cand + (Gq - 1) * kCandCap;           // selection: 128 values
      for (int x = lane; x < staged; x += 32) {
        const int j = x / k, e = x - j * k;
        st[x] = __ldcg(p.part_topk + ((piece_warp(j, Us, w0, T, W) + seg) * Gq + r) * k + e);
      }
      __syncwarp();
      float th = -INFINITY;
      for (int j = lane; j < np; j += 32) {
        float mn = INFINITY;
        for (int e = 0; e < k; ++e) mn = fminf(mn, st[j * k + e]);
        th = fmaxf(th, mn);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) th = fmaxf(th, __shfl_xor_sync(0xFFFFFFFFu, th, o));
      int count = 0;
      for (int xb = 0; xb < staged; xb += 32) {
        const int x = xb + lane;
        const float val = x < staged ? st[x] : -INFINITY;
        const bool keep = x < staged && val >= th && val > -INFINITY;
        const unsigned bal = __ballot_sync(0xFFFFFFFFu, keep);
        const int at = count + __popc(bal & ((1u << lane) - 1u));
        if (keep && at < kCandCap) sb[at] = val;
        count += __popc(bal);
      }
      __syncwarp();
      if (count <= kCandCap) {
#pragma unroll
        for (int j = 0; j < 4; ++j) v[j] = (lane * 4 + j < count) ? sb[lane * 4 + j] : -INFINITY;
        bitonic128_desc(v);
        done = true;
      }
      __syncwarp();
    }
    if (!done) {
      // general path: fold the lists in, one piece at a time
#pragma unroll
      for (int j = 0; j < 4; ++j) v[j] = -INFINITY;
      for (int j = 0; j < np; ++j) {
        const float* src = p.part_topk + ((piece_warp(j, Us, w0, T, W) + seg) * Gq + r) * k;
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          const int e = lane * 4 + x;
          if (e >= k) v[x] = (e < 2 * k) ? __ldcg(src + e - k) : -INFINITY;
        }
        bitonic128_desc(v);
      }
    }
    float sum = 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (lane * 4 + j < k) sum += exp2_approx(v[j] - M);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
    if (lane == 0) p.mass[row] = sum * inv;
  }
}

// Sequences with no live token: zeros (and mass 0), written by the grid.
__device__ void write_empty_outputs(const DecodeParams& p, const int32_t* P, int D) {
  const int64_t nthreads = (int64_t)gridDim.x * blockDim.x;
  const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  for (int64_t x = tid; x < (int64_t)p.n * p.Hq; x += nthreads) {
    const int i = (int)(x / p.Hq);
    if (P[i + 1] != P[i]) continue;
    uint16_t* o = p.out + x * D;
    for (int c = 0; c < D; ++c) o[c] = 0;
    if (p.mass) p.mass[x] = 0.f;
  }
}

// Per-warp state of the (sequence, kv-head) segment being processed.
template <int D, int G>
struct SegState {
  static constexpr int NG = D / G;
  static constexpr int KS = G / 16;   // k-steps per group
  static constexpr int MT = D / 16;   // m-tiles (16 channels) of the PV product
  float qsum[NG][2];                  // per-group sum of q for heads 2t, 2t+1
  float m[2], lp[2];                  // running max (log2 units), partial row sums
  float z[NG][2];                     // zero-term accumulators (heads 2t, 2t+1)
  float acc[MT][4];                   // PV accumulators (centred codes), units of 2^-sigma
  int sigma;                          // W = p * s_V * 2^sigma is the fp16 PV operand
};

template <int D, int G>
__device__ inline void seg_begin(SegState<D, G>& S, const DecodeParams& p, const uint16_t* qsm,
                                 uint2* qfrag, const TopkCtx& tk) {
  constexpr int NG = SegState<D, G>::NG, KS = SegState<D, G>::KS, MT = SegState<D, G>::MT;
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const bool has = g < p.Gq;
  const uint16_t* qrow = qsm + (has ? g : 0) * D;   // the segment's Gq query rows, in smem
  float qs[NG];
#pragma unroll
  for (int gr = 0; gr < NG; ++gr) {
    qs[gr] = 0.f;
#pragma unroll
    for (int s = 0; s < KS; ++s) {
      const uint16_t* qp = qrow + gr * G + t * (G / 4) + 4 * s;
      uint2 v = has ? *reinterpret_cast<const uint2*>(qp) : make_uint2(0, 0);
      qfrag[(gr * KS + s) * 32 + lane] = v;   // Q^T B-fragment of k-step (gr, s), head = gid
      __half2 a = *reinterpret_cast<__half2*>(&v.x), b = *reinterpret_cast<__half2*>(&v.y);
      float2 fa = __half22float2(a), fb = __half22float2(b);
      qs[gr] += (fa.x + fa.y) + (fb.x + fb.y);
    }
    qs[gr] += __shfl_xor_sync(0xFFFFFFFFu, qs[gr], 1);
    qs[gr] += __shfl_xor_sync(0xFFFFFFFFu, qs[gr], 2);
    S.qsum[gr][0] = __shfl_sync(0xFFFFFFFFu, qs[gr], 8 * t);
    S.qsum[gr][1] = __shfl_sync(0xFFFFFFFFu, qs[gr], 8 * t + 4);
    S.z[gr][0] = S.z[gr][1] = 0.f;
  }
  S.sigma = kSigmaInit;               // the first page sets sigma
  S.m[0] = S.m[1] = -INFINITY;
  S.lp[0] = S.lp[1] = 0.f;
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) S.acc[mt][0] = S.acc[mt][1] = S.acc[mt][2] = S.acc[mt][3] = 0.f;
  if (tk.topk > 0) {
    if (lane < p.Gq) {
      tk.cnt[lane] = 0;
      tk.theta[lane] = -INFINITY;
    }
    __syncwarp();
  }
}

template <int D, int G>
__device__ inline void seg_end(SegState<D, G>& S, const DecodeParams& p, int64_t piece,
                               const TopkCtx& tk, const int32_t* P, int i, int h, int64_t T,
                               int64_t W, float* scratch) {
  constexpr int NG = SegState<D, G>::NG, MT = SegState<D, G>::MT;
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    S.lp[0] += __shfl_xor_sync(0xFFFFFFFFu, S.lp[0], o);
    S.lp[1] += __shfl_xor_sync(0xFFFFFFFFu, S.lp[1], o);
#pragma unroll
    for (int gr = 0; gr < NG; ++gr) {
      S.z[gr][0] += __shfl_xor_sync(0xFFFFFFFFu, S.z[gr][0], o);
      S.z[gr][1] += __shfl_xor_sync(0xFFFFFFFFu, S.z[gr][1], o);
    }
  }
  const int Gq = p.Gq;
  float* po = p.part_o + piece * Gq * D;
  if (g == 0) {
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const int hd = 2 * t + c;
      if (hd < Gq) {
        p.part_ml[(piece * Gq + hd) * 2 + 0] = S.m[c];
        p.part_ml[(piece * Gq + hd) * 2 + 1] = S.lp[c];
      }
    }
  }
  const float inv = pow2i(-S.sigma);
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) {
    const int gr = (mt * 16) / G;
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      const int c = x & 1, ch = mt * 16 + g + 8 * (x >> 1), hd = 2 * t + c;
      if (hd < Gq) po[hd * D + ch] = fmaf(S.acc[mt][x], inv, S.z[gr][c]);
    }
  }
  if (tk.topk > 0) {
    for (int hd = 0; hd < Gq; ++hd) {
      if (tk.cnt[hd] > tk.topk) cand_compact(tk, hd);
      const int n = tk.cnt[hd];
      float* dst = p.part_topk + (piece * Gq + hd) * tk.topk;
      for (int j = lane; j < tk.topk; j += 32) dst[j] = j < n ? tk.cand[hd * kCandCap + j] : -INFINITY;
    }
    __syncwarp();
  }
  // arrival: the last warp to finish a piece of this segment merges all pieces
  const int nl = P[i + 1] - P[i];
  const int64_t Us = (int64_t)P[i] * p.Hkv + (int64_t)h * nl, Ue = Us + nl;
  const int64_t w0 = ((Us + 1) * W - 1) / T, w1 = (Ue * W - 1) / T;
  // with T <= W every non-empty warp holds exactly one unit; otherwise none is empty
  const uint32_t npieces = (uint32_t)(T <= W ? (int64_t)nl : w1 - w0 + 1);
  __threadfence();
  __syncwarp();
  uint32_t old = 0;
  if (lane == 0) old = atomicInc(&p.ctr[(int64_t)i * p.Hkv + h], npieces - 1);
  old = __shfl_sync(0xFFFFFFFFu, old, 0);
  if (old == npieces - 1) {
    __threadfence();
    merge_segment<D>(p, i, h, Us, w0, (int)npieces, T, W, tk, scratch);
  }
}

// One live page-head block (in shared memory) of a class with B-bit codes.
//   QK: S^T[16 slots x 8 heads] = K(codes) x Q^T per group, with codes as
//       fp16 (1024 + code); the 1024 offset folds into the group's zero term:
//       q.k = s * sum q (1024 + c) + (z - 1024 s) * sum q.
//   PV: O^T[16 channels x 8 heads] += V^T(codes - 2^(b-1)) x W per m-tile,
//       W = p * s_V * 2^sigma rounded to fp16, plus sum p (z + 2^(b-1) s) in fp32.
template <int D, int G, int B>
__device__ inline void page_step(SegState<D, G>& S, const uint8_t* blk, uint32_t mask,
                                 float scale_log2, float* pbuf, const TopkCtx& tk, int Gq) {
  const uint2* qfrag = reinterpret_cast<const uint2*>(reinterpret_cast<const uint8_t*>(pbuf) + kQfragOff);
  constexpr int NG = D / G, KS = G / 16, MT = D / 16;
  constexpr int LANE_BYTES = D * B / 16;
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const bool live0 = (mask >> g) & 1, live1 = (mask >> (g + 8)) & 1;
  const uint32_t* kpar = reinterpret_cast<const uint32_t*>(blk + 4 * D * B);      // [NG][16]
  const uint32_t* vpar = reinterpret_cast<const uint32_t*>(blk + 4 * D * B + 64 * NG);

  // ---------------- logits ----------------
  float lg[4] = {0.f, 0.f, 0.f, 0.f};
  {
    const uint8_t* kl = blk + lane * LANE_BYTES;
    constexpr int PB = G * B / 32;                        // piece bytes (>= 2)
    constexpr int NW = PB >= 4 ? PB / 4 : 1;              // words per piece
#pragma unroll
    for (int gr = 0; gr < NG; ++gr) {
      uint32_t w[2][NW];
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const uint8_t* src = kl + (gr * 2 + r) * PB;
        if constexpr (PB == 2) {
          const uint32_t h16 = *reinterpret_cast<const uint16_t*>(src);
          w[r][0] = (h16 & 0xFFu) | ((h16 & 0xFF00u) << 8);  // bytes -> half-words
        } else if constexpr (PB == 4) {
          w[r][0] = *reinterpret_cast<const uint32_t*>(src);
        } else if constexpr (PB == 8) {
          const uint2 v = *reinterpret_cast<const uint2*>(src);
          w[r][0] = v.x; w[r][1] = v.y;
        } else {
#pragma unroll
          for (int x = 0; x < PB / 16; ++x) {
            const uint4 v = *reinterpret_cast<const uint4*>(src + 16 * x);
            w[r][4 * x] = v.x; w[r][4 * x + 1] = v.y; w[r][4 * x + 2] = v.z; w[r][4 * x + 3] = v.w;
          }
        }
      }
      float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int s = 0; s < KS; ++s) {
        uint32_t a[4];
#pragma unroll
        for (int hi = 0; hi < 2; ++hi) {
          const int u = 2 * s + hi;                          // pair index inside the piece
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            if constexpr (B == 16) {
              a[hi * 2 + r] = w[r][u];
            } else {
              constexpr int PAIRS = (PB == 2 ? 4 : 16 / B);  // pairs per (spread) word
              a[hi * 2 + r] = unpack_pair<B>(w[r][u / PAIRS], u % PAIRS);
            }
          }
        }
        const uint2 qb = qfrag[(gr * KS + s) * 32 + lane];
        mma_16816(c, a, qb.x, qb.y);
      }
      if constexpr (B == 16) {
        lg[0] += c[0]; lg[1] += c[1]; lg[2] += c[2]; lg[3] += c[3];
      } else {
        const uint32_t p0 = kpar[gr * 16 + g], p1 = kpar[gr * 16 + g + 8];
        const float2 sz0 = __half22float2(*reinterpret_cast<const __half2*>(&p0));  // (s, z)
        const float2 sz1 = __half22float2(*reinterpret_cast<const __half2*>(&p1));
        const float zc0 = fmaf(-1024.f, sz0.x, sz0.y), zc1 = fmaf(-1024.f, sz1.x, sz1.y);
        lg[0] = fmaf(sz0.x, c[0], fmaf(zc0, S.qsum[gr][0], lg[0]));
        lg[1] = fmaf(sz0.x, c[1], fmaf(zc0, S.qsum[gr][1], lg[1]));
        lg[2] = fmaf(sz1.x, c[2], fmaf(zc1, S.qsum[gr][0], lg[2]));
        lg[3] = fmaf(sz1.x, c[3], fmaf(zc1, S.qsum[gr][1], lg[3]));
      }
    }
  }
  lg[0] = live0 ? lg[0] * scale_log2 : -INFINITY;
  lg[1] = live0 ? lg[1] * scale_log2 : -INFINITY;
  lg[2] = live1 ? lg[2] * scale_log2 : -INFINITY;
  lg[3] = live1 ? lg[3] * scale_log2 : -INFINITY;

  // ---------------- top-k candidates (logits above the head's threshold) ----------------
  if (tk.topk > 0) {
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      const int hd = 2 * t + (x & 1);
      if (hd < Gq && lg[x] > tk.theta[hd]) {
        const int at = atomicAdd(&tk.cnt[hd], 1);
        tk.cand[hd * kCandCap + at] = lg[x];
      }
    }
    __syncwarp();
    // a head whose buffer could overflow on the next page is cut back to its top-k
    unsigned full = __ballot_sync(0xFFFFFFFFu, lane < Gq && tk.cnt[lane] > kCandCap - 16);
    while (full) {
      cand_compact(tk, __ffs(full) - 1);
      full &= full - 1;
    }
  }

  // ---------------- online softmax (heads 2t, 2t+1) ----------------
  float pm0 = fmaxf(lg[0], lg[2]), pm1 = fmaxf(lg[1], lg[3]);
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    pm0 = fmaxf(pm0, __shfl_xor_sync(0xFFFFFFFFu, pm0, o));
    pm1 = fmaxf(pm1, __shfl_xor_sync(0xFFFFFFFFu, pm1, o));
  }
  const float mn0 = fmaxf(S.m[0], pm0), mn1 = fmaxf(S.m[1], pm1);
  const float a0 = exp2_approx(S.m[0] - mn0), a1 = exp2_approx(S.m[1] - mn1);
  S.m[0] = mn0;
  S.m[1] = mn1;
  float pr[4];
  pr[0] = exp2_approx(lg[0] - mn0);
  pr[1] = exp2_approx(lg[1] - mn1);
  pr[2] = exp2_approx(lg[2] - mn0);
  pr[3] = exp2_approx(lg[3] - mn1);
  S.lp[0] = fmaf(S.lp[0], a0, pr[0] + pr[2]);
  S.lp[1] = fmaf(S.lp[1], a1, pr[1] + pr[3]);

  if constexpr (B != 16) {
#pragma unroll
    for (int gr = 0; gr < NG; ++gr) {
      const uint32_t p0 = vpar[gr * 16 + g], p1 = vpar[gr * 16 + g + 8];
      const float2 sz0 = __half22float2(*reinterpret_cast<const __half2*>(&p0));
      const float2 sz1 = __half22float2(*reinterpret_cast<const __half2*>(&p1));
      const float zv0 = live0 ? fmaf((float)(1 << (B - 1)), sz0.x, sz0.y) : 0.f;
      const float zv1 = live1 ? fmaf((float)(1 << (B - 1)), sz1.x, sz1.y) : 0.f;
      S.z[gr][0] = fmaf(S.z[gr][0], a0, fmaf(pr[0], zv0, pr[2] * zv1));
      S.z[gr][1] = fmaf(S.z[gr][1], a1, fmaf(pr[1], zv0, pr[3] * zv1));
    }
  }

  // ---------------- p transpose: (tokens gid, gid+8 ; heads 2t, 2t+1) ->
  //                  (tokens 2t, 2t+1, 2t+8, 2t+9 ; head gid) ----------------
  *reinterpret_cast<float2*>(pbuf + g * kPbufStride + 2 * t) = make_float2(pr[0], pr[1]);
  *reinterpret_cast<float2*>(pbuf + (g + 8) * kPbufStride + 2 * t) = make_float2(pr[2], pr[3]);
  __syncwarp();
  float pt[4];
  pt[0] = pbuf[(2 * t) * kPbufStride + g];
  pt[1] = pbuf[(2 * t + 1) * kPbufStride + g];
  pt[2] = pbuf[(2 * t + 8) * kPbufStride + g];
  pt[3] = pbuf[(2 * t + 9) * kPbufStride + g];
  const uint32_t tmask = mask >> (2 * t);
  const bool tl[4] = {(tmask & 1u) != 0, (tmask & 2u) != 0, (tmask & 0x100u) != 0,
                      (tmask & 0x200u) != 0};

  // ---------------- PV operands W = p * s_V * 2^sigma (one sigma per segment) ----------------
  float sv[NG][4];
#pragma unroll
  for (int gr = 0; gr < NG; ++gr) {
    if constexpr (B == 16) {
      sv[gr][0] = sv[gr][1] = sv[gr][2] = sv[gr][3] = 1.f;
    } else {
      const uint2 q0 = *reinterpret_cast<const uint2*>(vpar + gr * 16 + 2 * t);
      const uint2 q1 = *reinterpret_cast<const uint2*>(vpar + gr * 16 + 2 * t + 8);
      sv[gr][0] = __half2float(__ushort_as_half((uint16_t)(q0.x & 0xFFFFu)));
      sv[gr][1] = __half2float(__ushort_as_half((uint16_t)(q0.y & 0xFFFFu)));
      sv[gr][2] = __half2float(__ushort_as_half((uint16_t)(q1.x & 0xFFFFu)));
      sv[gr][3] = __half2float(__ushort_as_half((uint16_t)(q1.y & 0xFFFFu)));
    }
  }
  // dead slots: p is 0, their scale bytes are stale; zero the packed operand instead
  const uint32_t dm0 = (tl[0] ? 0xFFFFu : 0u) | (tl[1] ? 0xFFFF0000u : 0u);
  const uint32_t dm1 = (tl[2] ? 0xFFFFu : 0u) | (tl[3] ? 0xFFFF0000u : 0u);
  float f = S.sigma == kSigmaInit ? 0.f : pow2i(S.sigma);
  float wv[NG][4];
  float wmax = 0.f;
#pragma unroll
  for (int gr = 0; gr < NG; ++gr)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      wv[gr][j] = pt[j] * f * sv[gr][j];
      wmax = tl[j] ? fmaxf(wmax, wv[gr][j]) : wmax;
    }
  float fac = 1.f;
  // slow path: first page of the segment, or a scale large enough to overflow fp16
  if (__any_sync(0xFFFFFFFFu, S.sigma == kSigmaInit || !(wmax < 32768.f))) {
    int e5 = 1;
#pragma unroll
    for (int gr = 0; gr < NG; ++gr)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int ef = (__float_as_int(sv[gr][j]) >> 23) - 112;  // fp16 exponent field
        e5 = tl[j] ? max(e5, ef) : e5;
      }
    e5 = max(e5, __shfl_xor_sync(0xFFFFFFFFu, e5, 1));
    e5 = max(e5, __shfl_xor_sync(0xFFFFFFFFu, e5, 2));
    const int sp = 29 - e5;             // s * 2^sp < 2^15 for every live scale of the page
    if (sp < S.sigma) {
      if (S.sigma != kSigmaInit) fac = pow2i(sp - S.sigma);
      S.sigma = sp;
    }
    f = pow2i(S.sigma);
#pragma unroll
    for (int gr = 0; gr < NG; ++gr)
#pragma unroll
      for (int j = 0; j < 4; ++j) wv[gr][j] = pt[j] * f * sv[gr][j];
  }
  uint32_t wf[NG][2];
#pragma unroll
  for (int gr = 0; gr < NG; ++gr) {
    wf[gr][0] = pack_half2_rn(wv[gr][0], wv[gr][1]) & dm0;
    wf[gr][1] = pack_half2_rn(wv[gr][2], wv[gr][3]) & dm1;
  }
  if (__any_sync(0xFFFFFFFFu, a0 != 1.f || a1 != 1.f || fac != 1.f)) {
    const float r0 = a0 * fac, r1 = a1 * fac;
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      S.acc[mt][0] *= r0;
      S.acc[mt][1] *= r1;
      S.acc[mt][2] *= r0;
      S.acc[mt][3] *= r1;
    }
  }

  // ---------------- O^T += V^T(codes - 2^(b-1)) x W ----------------
  {
    constexpr int Q = (B == 16) ? D / 8 : D * B / 128;   // words per token pair
    constexpr int PER = (B == 16) ? 1 : 16 / B;          // codes per half-word
    const uint32_t* vl = reinterpret_cast<const uint32_t*>(blk + 2 * D * B + lane * LANE_BYTES);
    // m-tiles in two halves (words q of P = 0 and P = 1 for half of the chunk
    // range); a single word per token pair (d = 64 at 2 bits) is one half
    constexpr int NHF = Q >= 2 ? 2 : 1;                    // halves
    constexpr int MH = MT / NHF;                           // m-tiles per half
    constexpr int QH = Q / NHF;                            // words per token pair per half
#pragma unroll
    for (int hf = 0; hf < NHF; ++hf) {
      uint32_t vr[2][QH];
#pragma unroll
      for (int P = 0; P < 2; ++P) {
        if constexpr (QH % 4 == 0) {
#pragma unroll
          for (int x = 0; x < QH / 4; ++x) {
            const uint4 v = reinterpret_cast<const uint4*>(vl + P * Q + hf * QH)[x];
            vr[P][4 * x] = v.x; vr[P][4 * x + 1] = v.y; vr[P][4 * x + 2] = v.z; vr[P][4 * x + 3] = v.w;
          }
        } else if constexpr (QH % 2 == 0) {
#pragma unroll
          for (int x = 0; x < QH / 2; ++x) {
            const uint2 v = reinterpret_cast<const uint2*>(vl + P * Q + hf * QH)[x];
            vr[P][2 * x] = v.x; vr[P][2 * x + 1] = v.y;
          }
        } else {
          vr[P][0] = vl[P * Q + hf * QH];
        }
      }
#pragma unroll
      for (int mh = 0; mh < MH; ++mh) {
        const int mt = hf * MH + mh;
        const int gr = (mt * 16) / G;
        uint32_t a[4];
#pragma unroll
        for (int P = 0; P < 2; ++P) {
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            const int e = 2 * mt + r;                       // element of L_g
            const int wq = e / PER - hf * QH;               // word within this half
            if constexpr (B == 16) {
              a[P * 2 + r] = vr[P][wq] & (P ? dm1 : dm0);   // raw values of dead slots: zero
            } else {
              // centred code pair c - 2^(b-1), exact in fp16: the sum over a
              // whole segment then carries no large offset to cancel
              a[P * 2 + r] = hsub2_bits(unpack_pair<B>(vr[P][wq], e % PER), centre_bits<B>());
            }
          }
        }
        mma_16816(S.acc[mt], a, wf[gr][0], wf[gr][1]);
      }
    }
  }
}

template <int D, int G>
__device__ inline void page_dispatch(SegState<D, G>& S, const uint8_t* blk, int bits, uint32_t mask,
                                     float scale_log2, float* pbuf, const TopkCtx& tk, int Gq) {
  switch (bits) {
    case 8: page_step<D, G, 8>(S, blk, mask, scale_log2, pbuf, tk, Gq); break;
    case 4: page_step<D, G, 4>(S, blk, mask, scale_log2, pbuf, tk, Gq); break;
    case 2: page_step<D, G, 2>(S, blk, mask, scale_log2, pbuf, tk, Gq); break;
    default: page_step<D, G, 16>(S, blk, mask, scale_log2, pbuf, tk, Gq); break;
  }
}

// What a lane knows about one unit (sequence, kv-head, live page): the page-head
// block's address, its class and segment (seg = i * Hkv + h), and the page's
// live mask.  The mask is loaded last and only needed once the page is computed.
struct UnitMeta {
  uint32_t src_lo, src_hi;
  uint32_t cls_seg;   // class << 24 | segment
  uint32_t mask;
};

__device__ inline UnitMeta resolve_unit(const DecodeParams& p, const int32_t* P, int64_t u,
                                        int64_t U1) {
  UnitMeta m;
  m.src_lo = m.src_hi = 0;
  m.cls_seg = 0;
  m.mask = 0;
  if (u >= U1) return m;
  int lo = 0, hi = p.n;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if ((int64_t)P[mid] * p.Hkv <= u) lo = mid; else hi = mid;
  }
  const int i = lo;
  const int nl = P[i + 1] - P[i];
  const int rel = (int)(u - (int64_t)P[i] * p.Hkv);   // < Hkv * max_blocks_per_seq < 2^31
  const int h = rel / nl, j = rel - h * nl;
  const int64_t row = (int64_t)p.seq[i] * p.max_blocks;
  const uint64_t desc = p.live_list[row + j];       // page | class << 32 | entry << 40
  const int cls = entry_class(desc);
  const uint64_t src = reinterpret_cast<uint64_t>(p.pool[cls]) +
                       ((uint64_t)entry_page(desc) * p.Hkv + h) * (uint64_t)p.phb[cls];
  m.src_lo = (uint32_t)src;
  m.src_hi = (uint32_t)(src >> 32);
  m.cls_seg = ((uint32_t)cls << 24) | (uint32_t)(i * p.Hkv + h);
  m.mask = entry_mask(p.table[row + live_desc_entry(desc)]);
  return m;
}

template <int D, int G>
__global__ void __launch_bounds__(kDecThreads, kDecMinBlocks)
    decode_split_kernel(DecodeParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int32_t* P = reinterpret_cast<int32_t*>(smem);

  // ---- prefix of live pages over the call's sequences (per CTA) ----
  {
    __shared__ int wsum[kDecWarps];
    int carry = 0;
    for (int base = 0; base < p.n; base += kDecThreads) {
      const int i = base + tid;
      int v = 0;
      if (i < p.n) {
        const int s = p.seq[i];
        if (s >= 0 && s < p.max_seqs) v = p.num_live[s];
        else if (blockIdx.x == 0) set_status(p.status, THINKV_ERR_INVALID);  // decoded as empty
      }
      int x = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xFFFFFFFFu, x, o);
        if (lane >= o) x += y;
      }
      if (lane == 31) wsum[warp] = x;
      __syncthreads();
      int before = carry;
      for (int w = 0; w < warp; ++w) before += wsum[w];
      if (i < p.n) P[i] = before + x - v;
      int tot = 0;
      for (int w = 0; w < kDecWarps; ++w) tot += wsum[w];
      carry += tot;
      __syncthreads();
    }
    if (tid == 0) P[p.n] = carry;
    __syncthreads();
  }
  write_empty_outputs(p, P, D);

  const int64_t T = (int64_t)P[p.n] * p.Hkv;
  const int64_t W = (int64_t)gridDim.x * kDecWarps;
  const int64_t w = (int64_t)blockIdx.x * kDecWarps + warp;
  const int64_t U0 = w * T / W, U1 = (w + 1) * T / W;
  if (U0 >= U1) return;

  uint8_t* wsm = smem + p.plan_smem + warp * p.warp_smem;
  uint64_t* bars = reinterpret_cast<uint64_t*>(wsm + p.nstage * p.stage_bytes);
  float* pbuf = reinterpret_cast<float*>(wsm + p.nstage * p.stage_bytes + 64);
  TopkCtx tk;
  {
    uint8_t* tb = wsm + p.nstage * p.stage_bytes + 64 + kPbufBytes;
    tk.cnt = reinterpret_cast<int*>(tb);
    tk.theta = reinterpret_cast<float*>(tb + 32);
    tk.cand = reinterpret_cast<float*>(tb + kTopkHdrBytes);
    tk.topk = p.topk;
  }
  if (lane == 0) {
    for (int s = 0; s < p.nstage; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
  }
  __syncwarp();

  UnitMeta cur = resolve_unit(p, P, U0 + lane, U1);
  UnitMeta nxt = resolve_unit(p, P, U0 + 32 + lane, U1);
  const int nu = (int)(U1 - U0);   // units of one warp: < 2^31

  // Issues unit ku (its lane in `m`) into stage st: the page-head block, plus
  // the segment's Q rows when ku is the first unit of a segment in this warp.
  int last_issued_seg = -1;
  auto issue = [&](const UnitMeta& m, int ku, int st) {
    const int srcl = ku & 31;
    const uint32_t lo = __shfl_sync(0xFFFFFFFFu, m.src_lo, srcl);
    const uint32_t hi = __shfl_sync(0xFFFFFFFFu, m.src_hi, srcl);
    const uint32_t cs = __shfl_sync(0xFFFFFFFFu, m.cls_seg, srcl);
    const int useg = (int)(cs & 0xFFFFFFu);
    const bool needq = useg != last_issued_seg;
    last_issued_seg = useg;
    if (lane == 0) {
      uint8_t* dst = wsm + st * p.stage_bytes;
      const uint32_t bytes = (uint32_t)p.phb[cs >> 24];
      mbar_arrive_expect_tx(&bars[st], bytes + (needq ? (uint32_t)p.q_bytes : 0u));
      bulk_g2s(dst, reinterpret_cast<const void*>(((uint64_t)hi << 32) | lo), bytes, &bars[st]);
      if (needq) {
        const int i = useg / p.Hkv, h = useg - (useg / p.Hkv) * p.Hkv;
        bulk_g2s(dst + p.q_off, p.q + ((int64_t)i * p.Hq + (int64_t)h * p.Gq) * D,
                 (uint32_t)p.q_bytes, &bars[st]);
      }
    }
  };

  // only the first page goes out before the loop: copies issued together all
  // land together, so the rest of the ring is filled once the first has landed
  issue(cur, 0, 0);

  SegState<D, G> S;
  int seg = -1;
  int stage = 0;
  uint32_t parity = 0;
  for (int k = 0; k < nu; ++k) {
    const int kk = k & 31;
    if (kk == 0 && k > 0) {
      cur = nxt;
      nxt = resolve_unit(p, P, U0 + k + 32 + lane, U1);
    }
    if (!mbar_wait_bounded(&bars[stage], parity)) {
      if (lane == 0) set_status(p.status, THINKV_ERR_TIMEOUT);
      // drain the copies still in flight (bounded), then leave
      const int issued = k == 0 ? 1 : min(nu, k + p.nstage);
      for (int k2 = k + 1; k2 < issued; ++k2)
        mbar_wait_bounded(&bars[k2 % p.nstage], (uint32_t)((k2 / p.nstage) & 1));
      return;
    }
    if (k == 0)
      for (int s2 = 1; s2 < p.nstage && s2 < nu; ++s2) issue(cur, s2, s2);
    const uint32_t cs = __shfl_sync(0xFFFFFFFFu, cur.cls_seg, kk);
    const int useg = (int)(cs & 0xFFFFFFu);
    uint8_t* blk = wsm + stage * p.stage_bytes;
    if (useg != seg) {
      if (seg >= 0) seg_end<D, G>(S, p, w + seg, tk, P, seg / p.Hkv, seg % p.Hkv, T, W, pbuf);
      seg = useg;
      seg_begin<D, G>(S, p, reinterpret_cast<const uint16_t*>(blk + p.q_off),
                      reinterpret_cast<uint2*>(reinterpret_cast<uint8_t*>(pbuf) + kQfragOff), tk);
      __syncwarp();
    }
    const uint32_t mask = __shfl_sync(0xFFFFFFFFu, cur.mask, kk);
    page_dispatch<D, G>(S, blk, p.bits[cs >> 24], mask & 0xFFFFu, p.scale_log2, pbuf, tk, p.Gq);
    __syncwarp();
    // refill this stage with unit k + nstage (from this batch of 32 or the next)
    const int kn = k + p.nstage;
    if (kn < nu) issue(((kn >> 5) == (k >> 5)) ? cur : nxt, kn, stage);
    if (++stage == p.nstage) {
      stage = 0;
      parity ^= 1u;
    }
  }
  if (seg >= 0) seg_end<D, G>(S, p, w + seg, tk, P, seg / p.Hkv, seg % p.Hkv, T, W, pbuf);
}

template <int D, int G>
cudaError_t launch_split(const DecodeParams& p, const DecodeLaunch& dl, cudaStream_t stream) {
  // raise the dynamic shared-memory limit of this instantiation once per device
  static size_t configured[64] = {0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (dl.smem_bytes > configured[dev]) {
    e = cudaFuncSetAttribute(decode_split_kernel<D, G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)dl.smem_bytes);
    if (e != cudaSuccess) return e;
    configured[dev] = dl.smem_bytes;
  }
  decode_split_kernel<D, G><<<dl.grid, kDecThreads, dl.smem_bytes, stream>>>(p);
  return cudaGetLastError();
}

int plan_smem_bytes(int32_t n) { return ((n + 1) * 4 + 127) / 128 * 128; }

}  // namespace

bool plan_decode_launch(const thinkv_layout& L, int32_t n_seqs, int32_t topk, int device,
                        DecodeLaunch* out) {
  const int D = L.head_dim, G = L.group_size;
  int64_t maxphb = 0;
  for (int c = 0; c < 3; ++c) {
    int64_t b = page_head_bytes(D, G, L.bits[c]);
    if (b > maxphb) maxphb = b;
  }
  const int Gq0 = L.num_q_heads / L.num_kv_heads;
  const int q_bytes = Gq0 * D * 2;
  const int stage_bytes = (int)((maxphb + 127) / 128 * 128) + (q_bytes + 127) / 128 * 128;
  // ~15 KB of page-head stages per warp keeps three 4-warp CTAs per SM
  int nstage = (int)(15360 / stage_bytes);
  if (nstage < 2) nstage = 2;
  if (nstage > 8) nstage = 8;
  const int Gq = L.num_q_heads / L.num_kv_heads;
  const int warp_smem = nstage * stage_bytes + 64 + kPbufBytes +
                        (topk > 0 ? kTopkHdrBytes + Gq * kCandCap * 4 : 0);
  const size_t smem = (size_t)plan_smem_bytes(n_seqs) + (size_t)kDecWarps * warp_smem;
  int optin = 0;
  if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, device) != cudaSuccess)
    return false;
  if (smem + 1024 > (size_t)optin) return false;
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device) != cudaSuccess) return false;
  int smem_per_sm = 0;
  if (cudaDeviceGetAttribute(&smem_per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, device) !=
      cudaSuccess)
    return false;
  // CTAs per SM: limited by shared memory (1 KB reserved per CTA) and by registers
  int per_sm = smem_per_sm / (int)(smem + 1024);
  int regs_per_sm = 0;
  if (cudaDeviceGetAttribute(&regs_per_sm, cudaDevAttrMaxRegistersPerMultiprocessor, device) !=
      cudaSuccess)
    return false;
  const int by_regs = regs_per_sm / (kDecRegs * kDecThreads);
  if (per_sm > by_regs) per_sm = by_regs;
  if (per_sm > 16) per_sm = 16;
  if (per_sm < 1) per_sm = 1;
  out->grid = sms * per_sm;
  out->warps_per_cta = kDecWarps;
  out->nstage = nstage;
  out->stage_bytes = stage_bytes;
  out->smem_bytes = smem;
  out->warp_smem = warp_smem;
  out->pieces = (int64_t)out->grid * kDecWarps + (int64_t)n_seqs * L.num_kv_heads;
  return true;
}

size_t decode_workspace_bytes(const thinkv_layout& L, int32_t n_seqs, int32_t topk,
                              const DecodeLaunch& dl) {
  const int Gq = L.num_q_heads / L.num_kv_heads;
  size_t b = ((size_t)n_seqs * L.num_kv_heads * 4 + 255) / 256 * 256;  // arrival counters
  b += ((size_t)dl.pieces * Gq * 2 * 4 + 255) / 256 * 256;
  b += ((size_t)dl.pieces * Gq * L.head_dim * 4 + 255) / 256 * 256;
  b += ((size_t)dl.pieces * Gq * (topk > 0 ? topk : 0) * 4 + 255) / 256 * 256;
  return b;
}

cudaError_t launch_decode(const CacheView& C, int32_t n, const int32_t* seq, const uint16_t* q,
                          uint16_t* out, float* mass, int32_t topk, float softmax_scale,
                          void* ws, const DecodeLaunch& dl, cudaStream_t stream) {
  const thinkv_layout& L = C.L;
  const int D = L.head_dim, G = L.group_size;
  DecodeParams p;
  for (int c = 0; c < 3; ++c) {
    p.pool[c] = C.pool[c];
    p.phb[c] = (int32_t)page_head_bytes(D, G, L.bits[c]);
    p.bits[c] = L.bits[c];
  }
  p.table = C.block_table;
  p.live_list = C.live_list;
  p.num_live = C.num_live;
  p.max_blocks = L.max_blocks_per_seq;
  p.max_seqs = L.max_seqs;
  p.Hkv = L.num_kv_heads;
  p.Hq = L.num_q_heads;
  p.Gq = L.num_q_heads / L.num_kv_heads;
  p.seq = seq;
  p.n = n;
  p.q = q;
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / sqrtf((float)D);
  p.scale_log2 = scale * 1.4426950408889634f;  // log2(e)
  uint8_t* w = static_cast<uint8_t*>(ws);
  p.ctr = reinterpret_cast<uint32_t*>(w);
  w += ((size_t)n * L.num_kv_heads * 4 + 255) / 256 * 256;
  p.part_ml = reinterpret_cast<float*>(w);
  w += ((size_t)dl.pieces * p.Gq * 2 * 4 + 255) / 256 * 256;
  p.part_o = reinterpret_cast<float*>(w);
  w += ((size_t)dl.pieces * p.Gq * D * 4 + 255) / 256 * 256;
  p.part_topk = reinterpret_cast<float*>(w);
  p.topk = mass ? topk : 0;
  p.live_count = C.live_count;
  p.out = out;
  p.mass = p.topk > 0 ? mass : nullptr;
  p.status = C.status;
  p.nstage = dl.nstage;
  p.stage_bytes = dl.stage_bytes;
  p.warp_smem = dl.warp_smem;
  {
    int64_t maxphb = 0;
    for (int c = 0; c < 3; ++c) maxphb = maxphb > p.phb[c] ? maxphb : p.phb[c];
    p.q_off = (int32_t)((maxphb + 127) / 128 * 128);
    p.q_bytes = p.Gq * D * 2;
  }
  p.plan_smem = plan_smem_bytes(n);
  cudaError_t e;
  if (D == 128 && G == 64) e = launch_split<128, 64>(p, dl, stream);
  else if (D == 128 && G == 32) e = launch_split<128, 32>(p, dl, stream);
  else if (D == 64 && G == 64) e = launch_split<64, 64>(p, dl, stream);
  else e = launch_split<64, 32>(p, dl, stream);
  return e;
}

}  // namespace thinkv
