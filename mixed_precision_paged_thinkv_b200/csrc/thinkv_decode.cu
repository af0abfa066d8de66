// thinkv_decode.cu -- decode attention over mixed-precision, slot-reusing pages.
//
// "ThinKV: Thought-Adaptive KV Cache Compression for Efficient Reasoning
// Models": the arXiv abstract's PagedAttention-based decode kernel, reading a
// cache whose tokens carry per-thought-type precision (explainer, Methodologie,
// TBQ) and whose evicted slots are holes that are never compacted (explainer,
// "Implementation Systeme: Pensee Continue (CT)").  The pages print no kernel
// design; this one is written for sm_100a:
//
//   One kernel per call.  The live page-heads of all decoded sequences form one
//   ordered list of units (sequence, kv-head, live page), segment by segment.
//   The grid has one CTA of 12 warps per SM; CTA c takes an equal contiguous
//   share of the units (stream-K at CTA level), and its warps split that
//   share into equal contiguous sub-ranges, so work is balanced by live pages
//   however lengths and budgets vary.  Per warp, lane 0 streams page-head
//   blocks (K codes, V codes, params: one contiguous block per page and head)
//   into a shared-memory ring with cp.async.bulk (TMA) + mbarriers, every
//   stage issued at once when the warp starts; the warp unpacks codes straight
//   into mma.sync m16n8k16 operands (byte-permute conversion to fp16 1024 +
//   code), computes q.k for the whole GQA group at once (tokens x heads),
//   applies the per-group scale/zero in fp32, runs the online softmax,
//   transposes p through a small shared buffer and accumulates p*scale (fp16,
//   exponent-shifted) times the centred V codes on the tensor cores, with the
//   zero terms summed in fp32.
//
//   A segment (sequence, kv-head) that lies wholly in one warp is written out
//   at once.  The others leave one piece (m, l, o, top-k logits) per warp;
//   after the loop the CTA merges the pieces of each of its segments with the
//   log-sum-exp rule (a warp per segment).  A segment that spans CTAs leaves
//   one piece per CTA in global memory; the last CTA to finish its piece
//   (a self-resetting arrival counter per segment) merges them and writes O
//   and the top-k mass.  Nothing waits on another CTA.
#include <cuda_fp16.h>
#include <limits.h>
#include <mutex>
#include <stdint.h>

#include "thinkv_common.cuh"
#include "thinkv_internal.h"

namespace thinkv {

namespace {

constexpr int kDecWarps = 12;                          // most warps per CTA (the plan may use fewer)
constexpr int kDecThreads = kDecWarps * 32;
constexpr int kDecMinBlocks = 1;                       // CTAs per SM the kernel is built for
constexpr int kPrefixPer = 4;                          // sequences per thread and prefix pass
constexpr int kPbufStride = 12;                 // floats per row of the p transpose buffer
// per-warp scratch: during pages, the p transpose (16 x 12 floats) and the
// segment's Q fragments (lane-contiguous, up to 2 KB); during a merge, after
// the loop, the weights of 32 pieces x 8 heads and the heads' M and L
constexpr int kPtBytes = 16 * kPbufStride * 4;          // 768
constexpr int kQfragOff = kPtBytes;
constexpr int kQfragBytes = 2048;                       // (D / 16) k-steps x 32 lanes x 8 B
constexpr int kPbufBytes = kPtBytes + kQfragBytes;      // >= 2 * 32 * 8 * 4 + 16 * 4
constexpr int kSigmaInit = 1 << 20;
constexpr int kMaxStages = 8;                   // page ring stages (one mbarrier each)
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
  uint32_t* cnt;     // [n * Hkv] arrival counters of segments spanning CTAs (zero between calls)
  uint8_t* wrec;     // [grid][nw] piece of each warp's first segment, when it is split
  uint8_t* crec;     // [grid][2] piece of each CTA's first / last segment, when it spans CTAs
  int32_t rb;        // bytes of one piece record
  const int32_t* live_count;
  uint16_t* out;     // [n][Hq][D]
  float* mass;       // [n][Hq] or null
  int32_t topk;
  int32_t* status;
  int32_t nw;        // warps per CTA (blockDim.x / 32)
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

// Sorts 64 values held 2 per lane (element lane*2 + j) into descending order.
__device__ inline void bitonic64_desc(float (&v)[2]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int size = 2; size <= 64; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      if (stride >= 2) {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int i = lane * 2 + j;
          const float o = __shfl_xor_sync(0xFFFFFFFFu, v[j], stride >> 1);
          const bool desc = (i & size) == 0, lower = (i & stride) == 0;
          v[j] = (lower == desc) ? fmaxf(v[j], o) : fminf(v[j], o);
        }
      } else {
        const bool desc = ((lane * 2) & size) == 0;
        const float a = v[0], b = v[1];
        v[0] = desc ? fmaxf(a, b) : fminf(a, b);
        v[1] = desc ? fminf(a, b) : fmaxf(a, b);
      }
    }
  }
}

// Sorts one value per lane into descending order across the warp.
__device__ inline float bitonic32_desc(float v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      const float o = __shfl_xor_sync(0xFFFFFFFFu, v, stride);
      const bool desc = (lane & size) == 0, lower = (lane & stride) == 0;
      v = (lower == desc) ? fmaxf(v, o) : fminf(v, o);
    }
  }
  return v;
}

struct TopkCtx {
  float* cand;    // [Gq][kCandCap]
  int* cnt;       // [Gq]
  float* theta;   // [Gq]  values <= theta cannot enter the top-k any more
  int topk;
};

// Cuts head h's candidates back to a few more than topk, without sorting
// them.  Needs topk <= 32 and at least 32 candidates, so that every lane holds
// one (candidate e sits at lane e % 32).  The lane maxima are sorted; the
// threshold is the largest of them with at least topk candidates at or above
// it (the topk-th largest lane maximum always qualifies).  Candidates below it
// are dropped: at least topk larger ones remain, so none of them can be among
// the topk largest.
__device__ inline void cand_prune(const TopkCtx& tk, int h) {
  const int lane = threadIdx.x & 31;
  float* c = tk.cand + h * kCandCap;
  const int n = tk.cnt[h];
  float v[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) v[j] = (j * 32 + lane < n) ? c[j * 32 + lane] : -INFINITY;
  const float s = bitonic32_desc(fmaxf(fmaxf(v[0], v[1]), fmaxf(v[2], v[3])));
  int lo = 0, hi = tk.topk - 1;                    // the answer lies in [lo, hi]
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    const float t = __shfl_sync(0xFFFFFFFFu, s, mid);
    int cnt = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) cnt += __popc(__ballot_sync(0xFFFFFFFFu, v[j] >= t));
    if (cnt >= tk.topk) hi = mid; else lo = mid + 1;
  }
  const float theta = __shfl_sync(0xFFFFFFFFu, s, lo);
  int kc = 0;
#pragma unroll
  for (int j = 0; j < 4; ++j) kc += v[j] >= theta;
  int incl = kc;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (lane >= o) incl += y;
  }
  const int kept = __shfl_sync(0xFFFFFFFFu, incl, 31);
  int at = incl - kc;
  __syncwarp();                                    // every read of c is done
#pragma unroll
  for (int j = 0; j < 4; ++j)
    if (v[j] >= theta) c[at++] = v[j];
  __syncwarp();
  if (lane == 0) {
    tk.cnt[h] = kept;
    tk.theta[h] = theta;
  }
  __syncwarp();
}

// Keeps the topk largest candidates of head h and raises its threshold.
__device__ inline void cand_compact(const TopkCtx& tk, int h) {
  const int lane = threadIdx.x & 31;
  float* c = tk.cand + h * kCandCap;
  const int n = tk.cnt[h];
  if (n <= 64) {
    // the smaller network suffices
    float u[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) u[j] = (lane * 2 + j < n) ? c[lane * 2 + j] : -INFINITY;
    bitonic64_desc(u);
    __syncwarp();
    const int keep = min(n, tk.topk);
#pragma unroll
    for (int j = 0; j < 2; ++j)
      if (lane * 2 + j < keep) c[lane * 2 + j] = u[j];
    const int kl = tk.topk - 1;
    const float kth = __shfl_sync(0xFFFFFFFFu, (kl & 1) ? u[1] : u[0], (kl >> 1) & 31);
    __syncwarp();
    if (lane == 0) {
      tk.cnt[h] = keep;
      if (n >= tk.topk) tk.theta[h] = kth;
    }
    __syncwarp();
    return;
  }
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

// ---------------------------------------------------------------------------
// partial results of split segments
// ---------------------------------------------------------------------------
// A piece of a (sequence, kv-head) segment is one contiguous record, so that a
// merge can fetch it with a single bulk copy:
//   [0, 64)                 (m, l) of query heads 0..7 (m in log2 units, l the
//                           row sum relative to m)
//   [64, 64 + 4*Gq*D)       the unnormalised output rows o[Gq][D]
//   then 4*Gq*kpad bytes    per head, the top-k largest logits, descending,
//                           -inf padded (kpad = topk rounded up to 4)
__host__ __device__ inline int64_t record_bytes(int Gq, int D, int topk) {
  const int kpad = (topk + 3) / 4 * 4;
  return 64 + 4LL * Gq * D + 4LL * Gq * kpad;
}

// Merges a bitonic sequence of 128 values held 4 per lane (element lane*4+j)
// into descending order.
__device__ inline void bitonic128_merge_desc(float (&v)[4]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int stride = 64; stride > 0; stride >>= 1) {
    if (stride >= 4) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float o = __shfl_xor_sync(0xFFFFFFFFu, v[j], stride >> 2);
        const bool lower = ((lane * 4 + j) & stride) == 0;
        v[j] = lower ? fmaxf(v[j], o) : fminf(v[j], o);
      }
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (j & stride) continue;
        const float x = v[j], y = v[j | stride];
        v[j] = fmaxf(x, y);
        v[j | stride] = fminf(x, y);
      }
    }
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
  float th[2];                        // top-k thresholds of heads 2t, 2t+1 (copies)
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
  S.th[0] = S.th[1] = -INFINITY;
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

// Unit range [Us, Ue) of segment (i, h) in the call's list of live page-heads.
__device__ inline void seg_range(const DecodeParams& p, const int32_t* P, int i, int h,
                                 int64_t* Us, int64_t* Ue) {
  const int nl = P[i + 1] - P[i];
  *Us = (int64_t)P[i] * p.Hkv + (int64_t)h * nl;
  *Ue = *Us + nl;
}

// Which of W equal contiguous shares of [0, T) (share w holds [w*T/W,
// (w+1)*T/W)) holds unit u < T.
__device__ inline int64_t share_of_unit(int64_t u, int64_t T, int64_t W) {
  return ((u + 1) * W - 1) / T;
}

// Ends the warp's work on segment seg = i * Hkv + h.  With piece == null the
// whole segment was in this warp: its O rows and top-k mass are written at
// once.  Otherwise the warp's piece record (m, l, unnormalised o, sorted top-k
// logits) is written at `piece` (shared or global memory) for the merge.
template <int D, int G>
__device__ inline void seg_end(SegState<D, G>& S, const DecodeParams& p, int seg,
                               const TopkCtx& tk, uint8_t* piece) {
  constexpr int NG = SegState<D, G>::NG, MT = SegState<D, G>::MT;
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int i = seg / p.Hkv, h = seg - (seg / p.Hkv) * p.Hkv;
  const bool whole = piece == nullptr;
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
  const float sinv = pow2i(-S.sigma);
  float* po = whole ? nullptr : reinterpret_cast<float*>(piece + 64);
  const float li0 = whole ? 1.f / S.lp[0] : 1.f, li1 = whole ? 1.f / S.lp[1] : 1.f;
  if (!whole && g == 0) {
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const int hd = 2 * t + c;
      if (hd < Gq) reinterpret_cast<float2*>(piece)[hd] = make_float2(S.m[c], S.lp[c]);
    }
  }
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) {
    const int gr = (mt * 16) / G;
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      const int c = x & 1, ch = mt * 16 + g + 8 * (x >> 1), hd = 2 * t + c;
      if (hd < Gq) {
        const float o = fmaf(S.acc[mt][x], sinv, S.z[gr][c]);
        if (whole)
          p.out[((int64_t)i * p.Hq + h * Gq + hd) * D + ch] =
              __half_as_ushort(__float2half_rn(o * (c ? li1 : li0)));
        else
          po[hd * D + ch] = o;
      }
    }
  }
  if (tk.topk > 0) {
    const int kpad = (tk.topk + 3) / 4 * 4;
    const bool all = whole && p.live_count[__ldg(p.seq + i)] <= tk.topk;
    float* tl = whole ? nullptr : reinterpret_cast<float*>(piece + 64 + 4 * Gq * D);
    for (int hd = 0; hd < Gq; ++hd) {
      float sum = 0.f;
      if (!all) {
        if (tk.topk <= 32 && tk.cnt[hd] > 64) cand_prune(tk, hd);   // then the 64-wide sort
        if (tk.cnt[hd] > 0) cand_compact(tk, hd);      // sorted, the k largest kept
        const int n = tk.cnt[hd];
        if (whole) {
          const float m = __shfl_sync(0xFFFFFFFFu, (hd & 1) ? S.m[1] : S.m[0], hd >> 1);
          for (int j = lane; j < n; j += 32) sum += exp2_approx(tk.cand[hd * kCandCap + j] - m);
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
        } else {
          for (int j = lane; j < kpad; j += 32)
            tl[hd * kpad + j] = j < n ? tk.cand[hd * kCandCap + j] : -INFINITY;
        }
      }
      if (whole) {
        const float l = __shfl_sync(0xFFFFFFFFu, (hd & 1) ? S.lp[1] : S.lp[0], hd >> 1);
        if (lane == 0) p.mass[(int64_t)i * p.Hq + h * Gq + hd] = all ? 1.f : sum / l;
      }
    }
  }
  __syncwarp();
}

// Words [w0, w0 + NW) of this lane's portion of a code region laid out in
// chunks of U = min(16, LB) bytes interleaved over the 32 lanes (see
// lane_off); `base` is the region + lane * U.  w0 and NW are multiples of U/4,
// so every load is one whole chunk: 32 lanes read one contiguous span.
template <int LB, int NW>
__device__ __forceinline__ void lane_words(const uint8_t* base, int w0, uint32_t (&dst)[NW]) {
  constexpr int U = LB < 16 ? LB : 16;
#pragma unroll
  for (int x = 0; x < NW; x += U / 4) {
    const uint8_t* ptr = base + ((w0 + x) * 4 / U) * 32 * U;
    if constexpr (U == 16) {
      const uint4 v = *reinterpret_cast<const uint4*>(ptr);
      dst[x] = v.x; dst[x + 1] = v.y; dst[x + 2] = v.z; dst[x + 3] = v.w;
    } else {
      const uint2 v = *reinterpret_cast<const uint2*>(ptr);
      dst[x] = v.x; dst[x + 1] = v.y;
    }
  }
}

// One live page-head block (in shared memory) of a class with B-bit codes.
//   QK: S^T[16 slots x 8 heads] = K(codes) x Q^T per group.  8-bit codes enter
//       as fp16 (1024 + code) and the offset folds into the group's zero term:
//       q.k = s * sum q (1024 + c) + (z - 1024 s) * sum q.  4- and 2-bit codes
//       have scales large enough that the cancellation of the 1024 s term
//       would cost precision: they enter centred, (code - 2^(b-1)), exactly,
//       and q.k = s * sum q (c - 2^(b-1)) + (z + 2^(b-1) s) * sum q.
//   PV: O^T[16 channels x 8 heads] += V^T(codes - 2^(b-1)) x W per m-tile,
//       W = p * s_V * 2^sigma rounded to fp16, plus sum p (z + 2^(b-1) s) in fp32.
//       8-bit codes: the MMA takes (1024 + code) and a constant-row product
//       removes the offset; 4- and 2-bit codes are centred in the operand (a
//       centred code of 1 or 2 next to a 1024 offset would lose 9-10 bits of
//       the running accumulator on every page).
//   Float codes (FP8 E4M3 at b = 8, FP4 E2M1 at b = 4; F = 1) enter as their
//   exact fp16 values with no offset and a zero of 0; ternary codes are the
//   2-bit integer path (zero = -scale).
template <int D, int G, int B, int F = 0>
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
    constexpr int U = LANE_BYTES < 16 ? LANE_BYTES : 16;
    const uint8_t* kbase = blk + lane * U;
    constexpr int PB = G * B / 32;                        // piece bytes (>= 2)
    constexpr int NW = PB >= 4 ? PB / 4 : 1;              // words per piece
    // a lane portion of up to 32 bytes is loaded whole, a larger one per group
    constexpr bool KALL = LANE_BYTES <= 32;
    constexpr int KW = KALL ? LANE_BYTES / 4 : 2 * PB / 4;
    uint32_t kw[KW];
    if constexpr (KALL) lane_words<LANE_BYTES, KW>(kbase, 0, kw);
#pragma unroll
    for (int gr = 0; gr < NG; ++gr) {
      if constexpr (!KALL) lane_words<LANE_BYTES, KW>(kbase, gr * 2 * PB / 4, kw);
      uint32_t w[2][NW];
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        if constexpr (PB == 2) {
          const uint32_t h16 = (kw[gr] >> (16 * r)) & 0xFFFFu;   // piece 2 gr + r
          w[r][0] = (h16 & 0xFFu) | ((h16 & 0xFF00u) << 8);  // bytes -> half-words
        } else {
#pragma unroll
          for (int x = 0; x < NW; ++x) w[r][x] = kw[(KALL ? gr * 2 * NW : 0) + r * NW + x];
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
              if constexpr (F == 1) {
                a[hi * 2 + r] = unpack_float_pair<B>(w[r][u / PAIRS], u % PAIRS);
              } else {
                a[hi * 2 + r] = unpack_pair<B>(w[r][u / PAIRS], u % PAIRS);
                if constexpr (B != 8) a[hi * 2 + r] = hsub2_bits(a[hi * 2 + r], centre_bits<B>());
              }
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
        constexpr float off = F == 1 ? 0.f : (B == 8 ? -1024.f : (float)(1 << (B - 1)));   // see above
        const float zc0 = fmaf(off, sz0.x, sz0.y), zc1 = fmaf(off, sz1.x, sz1.y);
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
    // the thresholds are register copies; they change only when a buffer is cut
    bool ins = false;
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      const int hd = 2 * t + (x & 1);
      if (hd < Gq && lg[x] > S.th[x & 1]) {
        const int at = atomicAdd(&tk.cnt[hd], 1);
        tk.cand[hd * kCandCap + at] = lg[x];
        ins = true;
      }
    }
    if (__any_sync(0xFFFFFFFFu, ins)) {
      __syncwarp();
      // a head whose buffer could overflow on the next page is cut back
      unsigned full = __ballot_sync(0xFFFFFFFFu, lane < Gq && tk.cnt[lane] > kCandCap - 16);
      if (full) {
        while (full) {
          const int hf = __ffs(full) - 1;
          if (tk.topk <= 32) cand_prune(tk, hf);
          // ties can keep too many: then the exact cut, which keeps topk
          if (tk.cnt[hf] > kCandCap - 16) cand_compact(tk, hf);
          full &= full - 1;
        }
        S.th[0] = 2 * t < Gq ? tk.theta[2 * t] : INFINITY;
        S.th[1] = 2 * t + 1 < Gq ? tk.theta[2 * t + 1] : INFINITY;
      }
    }
  }

  // ---------------- online softmax (heads 2t, 2t+1) ----------------
  // Most pages raise no head's running max: the max over the page's tokens is
  // only formed (and the rescale factors with it) when some logit exceeds it.
  float a0 = 1.f, a1 = 1.f;
  float mn0 = S.m[0], mn1 = S.m[1];
  if (__any_sync(0xFFFFFFFFu, fmaxf(lg[0], lg[2]) > mn0 || fmaxf(lg[1], lg[3]) > mn1)) {
    float pm0 = fmaxf(lg[0], lg[2]), pm1 = fmaxf(lg[1], lg[3]);
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      pm0 = fmaxf(pm0, __shfl_xor_sync(0xFFFFFFFFu, pm0, o));
      pm1 = fmaxf(pm1, __shfl_xor_sync(0xFFFFFFFFu, pm1, o));
    }
    mn0 = fmaxf(S.m[0], pm0);
    mn1 = fmaxf(S.m[1], pm1);
    a0 = exp2_approx(S.m[0] - mn0);
    a1 = exp2_approx(S.m[1] - mn1);
    S.m[0] = mn0;
    S.m[1] = mn1;
  }
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
      constexpr float voff = F == 1 ? 0.f : (float)(1 << (B - 1));
      const float zv0 = live0 ? fmaf(voff, sz0.x, sz0.y) : 0.f;
      const float zv1 = live1 ? fmaf(voff, sz1.x, sz1.y) : 0.f;
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

  // ---------------- O^T += V^T(codes - 2^(b-1)) x W, per m-tile (8-bit: V^T(1024 + codes) x W
  //                  plus one constant-row product that removes 1024 + 2^(b-1)) ----------------
  {
    constexpr int Q = (B == 16) ? D / 8 : D * B / 128;   // words per token pair
    constexpr int PER = (B == 16) ? 1 : 16 / B;          // codes per half-word
    constexpr int U = LANE_BYTES < 16 ? LANE_BYTES : 16;
    const uint8_t* vbase = blk + 2 * D * B + lane * U;
    // a lane portion of up to 32 bytes is loaded whole, a larger one per half
    constexpr bool VALL = LANE_BYTES <= 32;
    uint32_t vall[VALL ? LANE_BYTES / 4 : 1];
    if constexpr (VALL) lane_words<LANE_BYTES, (VALL ? LANE_BYTES / 4 : 1)>(vbase, 0, vall);
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
        if constexpr (VALL) {
#pragma unroll
          for (int x = 0; x < QH; ++x) vr[P][x] = vall[P * Q + hf * QH + x];
        } else {
          lane_words<LANE_BYTES, QH>(vbase, P * Q + hf * QH, vr[P]);
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
              if constexpr (F == 1) {
                // value(code); a dead slot's stale byte may be an E4M3 NaN,
                // which its zero weight would not cancel: zero it here
                a[P * 2 + r] = unpack_float_pair<B>(vr[P][wq], e % PER) & (P ? dm1 : dm0);
              } else {
                a[P * 2 + r] = unpack_pair<B>(vr[P][wq], e % PER);   // 1024 + code
                if constexpr (B != 8) a[P * 2 + r] = hsub2_bits(a[P * 2 + r], centre_bits<B>());
              }
            }
          }
        }
        mma_16816(S.acc[mt], a, wf[gr][0], wf[gr][1]);
        if constexpr (B == 8 && F == 0) {
          // centre at once: + (-(1024 + 2^(b-1))) * sum of W over the page's
          // tokens, so the segment's accumulators never carry the offset
          const uint32_t kc = neg_centre_bits<B>();
          const uint32_t ka[4] = {kc, kc, kc, kc};
          mma_16816(S.acc[mt], ka, wf[gr][0], wf[gr][1]);
        }
      }
    }
  }
}

// bits: the class's code width, plus 256 for the float formats at 8 and 4 bits
template <int D, int G>
__device__ inline void page_dispatch(SegState<D, G>& S, const uint8_t* blk, int bits, uint32_t mask,
                                     float scale_log2, float* pbuf, const TopkCtx& tk, int Gq) {
  switch (bits) {
    case 256 + 8: page_step<D, G, 8, 1>(S, blk, mask, scale_log2, pbuf, tk, Gq); break;
    case 256 + 4: page_step<D, G, 4, 1>(S, blk, mask, scale_log2, pbuf, tk, Gq); break;
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

// Call index i whose units hold unit u (P: prefix of live pages, n + 1 entries).
__device__ inline int seq_of_unit(const DecodeParams& p, const int32_t* P, int64_t u) {
  int lo = 0, hi = p.n;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if ((int64_t)P[mid] * p.Hkv <= u) lo = mid; else hi = mid;
  }
  return lo;
}

// Segment (i * Hkv + h) of unit u.
__device__ inline int seg_of_unit(const DecodeParams& p, const int32_t* P, int64_t u) {
  const int i = seq_of_unit(p, P, u);
  const int nl = P[i + 1] - P[i];
  return i * p.Hkv + (int)((u - (int64_t)P[i] * p.Hkv) / nl);
}

__device__ inline UnitMeta resolve_unit(const DecodeParams& p, const int32_t* P, int64_t u,
                                        int64_t U1) {
  UnitMeta m;
  m.src_lo = m.src_hi = 0;
  m.cls_seg = 0;
  m.mask = 0;
  if (u >= U1) return m;
  const int i = seq_of_unit(p, P, u);
  const int nl = P[i + 1] - P[i];
  const int rel = (int)(u - (int64_t)P[i] * p.Hkv);   // < Hkv * max_blocks_per_seq < 2^31
  const int h = rel / nl, j = rel - h * nl;
  const int64_t row = (int64_t)__ldg(p.seq + i) * p.max_blocks;
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

// ---------------------------------------------------------------------------
// merging the pieces of one segment (the whole CTA)
// ---------------------------------------------------------------------------
// Loads of piece records: records written by other CTAs are read through L2
// (kL2); the CTA's own records (shared memory, or global memory written by
// its warps before a __syncthreads) with ordinary loads.
template <bool kL2, typename T>
__device__ __forceinline__ T ld_rec(const T* ptr) {
  if constexpr (kL2) return __ldcg(ptr);
  else return *ptr;
}

// Merges np piece records of segment `seg` with the log-sum-exp rule (one
// warp): per head, M = max m_j, L = sum l_j 2^(m_j - M), o = sum o_j
// 2^(m_j - M), and the top-k logits of all pieces merged into one sorted
// list.  If dst is null the result is final: O = o / L in fp16 and the top-k
// mass are written out.  Otherwise the merged piece is written at dst (a
// record, for a later merge).  `piece(j)` gives the address of record j.
// Written for few memory round trips: the (m, l) pairs of up to 16 pieces
// are requested at once into a shared table, every lane requests all its
// output quads of a piece at once, and each head's top-k lists are staged in
// shared memory with one pass of loads before the bitonic merges.
// wb: this warp's 704-float scratch: M[8], L[8], ints [16, 176) for the
// caller's piece list, the table at [176, 432), weights at [432, 560); the
// top-k staging reuses [176, 704).
template <int D, bool kL2, typename PieceFn>
__device__ void merge_pieces(const DecodeParams& p, int seg, int np, PieceFn piece, uint8_t* dst,
                             float* wb) {
  const int lane = threadIdx.x & 31;
  const int Gq = p.Gq, k = p.topk, kpad = (k + 3) / 4 * 4;
  const int i = seg / p.Hkv, h = seg - (seg / p.Hkv) * p.Hkv;
  constexpr int CH = 16;                          // pieces per table chunk
  float* M = wb;
  float* L = wb + 8;
  float2* tbl = reinterpret_cast<float2*>(wb + 176);
  float* wt = wb + 432;
  auto load_table = [&](int j0, int cnt) {
    for (int x = lane; x < cnt * Gq; x += 32) {
      const int j = x / Gq, r = x - j * Gq;
      tbl[j * 8 + r] = ld_rec<kL2>(reinterpret_cast<const float2*>(piece(j0 + j)) + r);
    }
    __syncwarp();
  };
  // maxima (one chunk: the table stays for the weights)
  if (lane < 8) {
    M[lane] = -INFINITY;
    L[lane] = 0.f;
  }
  for (int j0 = 0; j0 < np; j0 += CH) {
    load_table(j0, min(CH, np - j0));
    if (lane < Gq) {
      float m = M[lane];
      for (int j = 0; j < min(CH, np - j0); ++j) m = fmaxf(m, tbl[j * 8 + lane].x);
      M[lane] = m;
    }
    __syncwarp();
  }
  constexpr int QD = D / 4;
  const int nquad = Gq * QD;                      // <= 256: at most 8 quads per lane
  float4 acc[8];
#pragma unroll
  for (int x = 0; x < 8; ++x) acc[x] = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int j0 = 0; j0 < np; j0 += CH) {
    const int cnt = min(CH, np - j0);
    if (np > CH) load_table(j0, cnt);             // else the table is still there
    if (lane < Gq) {                              // weights, and L in a fixed order
      float l = L[lane];
      for (int j = 0; j < cnt; ++j) {
        const float2 ml = tbl[j * 8 + lane];
        const float w = ml.x == -INFINITY ? 0.f : exp2_approx(ml.x - M[lane]);
        wt[j * 8 + lane] = w;
        l = fmaf(w, ml.y, l);
      }
      L[lane] = l;
    }
    __syncwarp();
    for (int j = 0; j < cnt; ++j) {               // a piece's quads all in flight
      const float4* o = reinterpret_cast<const float4*>(piece(j0 + j) + 64);
      float4 v[8];
#pragma unroll
      for (int x = 0; x < 8; ++x) {
        const int e = x * 32 + lane;
        if (e < nquad) v[x] = ld_rec<kL2>(o + e);
      }
#pragma unroll
      for (int x = 0; x < 8; ++x) {
        const int e = x * 32 + lane;
        if (e < nquad) {
          const float w = wt[j * 8 + e / QD];
          acc[x].x = fmaf(w, v[x].x, acc[x].x);
          acc[x].y = fmaf(w, v[x].y, acc[x].y);
          acc[x].z = fmaf(w, v[x].z, acc[x].z);
          acc[x].w = fmaf(w, v[x].w, acc[x].w);
        }
      }
    }
    __syncwarp();                                 // the weights are refilled by the next chunk
  }
#pragma unroll
  for (int x = 0; x < 8; ++x) {
    const int e = x * 32 + lane;
    if (e >= nquad) continue;
    const int r = e / QD, q4 = e - r * QD;
    if (dst == nullptr) {
      const float inv = 1.f / L[r];
      const uint32_t lo = (uint32_t)__half_as_ushort(__float2half_rn(acc[x].x * inv)) |
                          ((uint32_t)__half_as_ushort(__float2half_rn(acc[x].y * inv)) << 16);
      const uint32_t hi = (uint32_t)__half_as_ushort(__float2half_rn(acc[x].z * inv)) |
                          ((uint32_t)__half_as_ushort(__float2half_rn(acc[x].w * inv)) << 16);
      const int64_t row = (int64_t)i * p.Hq + h * Gq + r;
      reinterpret_cast<uint2*>(p.out + row * D)[q4] = make_uint2(lo, hi);
    } else {
      reinterpret_cast<float4*>(dst + 64)[e] = acc[x];
    }
  }
  if (dst != nullptr && lane < Gq) reinterpret_cast<float2*>(dst)[lane] = make_float2(M[lane], L[lane]);
  if (k > 0) {
    const bool all = dst == nullptr && p.live_count[__ldg(p.seq + i)] <= k;
    float* stage = wb + 176;
    const int per = (704 - 176) / kpad;            // lists one staging pass holds
    for (int r = 0; r < Gq; ++r) {
      if (all) {
        if (lane == 0) p.mass[(int64_t)i * p.Hq + h * Gq + r] = 1.f;
        continue;
      }
      // running list (descending) in elements 0..63, the next piece's list
      // reversed in 64..127: a bitonic sequence
      float tv[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) tv[e] = -INFINITY;
      for (int j0 = 0; j0 < np; j0 += per) {
        const int cnt = min(per, np - j0);
        __syncwarp();
        for (int x = lane; x < cnt * kpad; x += 32) {
          const int j = x / kpad, m = x - j * kpad;
          stage[x] = ld_rec<kL2>(reinterpret_cast<const float*>(piece(j0 + j) + 64 + 4 * Gq * D) +
                                 r * kpad + m);
        }
        __syncwarp();
        for (int j = 0; j < cnt; ++j) {
          float v[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int el = lane * 4 + e, m = 127 - el;
            v[e] = el < 64 ? tv[e] : (m < k ? stage[j * kpad + m] : -INFINITY);
          }
          bitonic128_merge_desc(v);
#pragma unroll
          for (int e = 0; e < 4; ++e) tv[e] = v[e];
        }
      }
      if (dst == nullptr) {
        float sum = 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (lane * 4 + e < k) sum += exp2_approx(tv[e] - M[r]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
        if (lane == 0) p.mass[(int64_t)i * p.Hq + h * Gq + r] = sum / L[r];
      } else {
        float* tl = reinterpret_cast<float*>(dst + 64 + 4 * Gq * D) + r * kpad;
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (lane * 4 + e < kpad) tl[lane * 4 + e] = tv[e];
      }
    }
  }
  __syncwarp();
}

template <int D, int G>
__global__ void __launch_bounds__(kDecThreads, kDecMinBlocks) decode_kernel(DecodeParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ int wsum[kDecWarps];
  __shared__ int s_last[kDecWarps];                // each warp's last segment
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int NW = p.nw, NT = NW * 32;
  int32_t* P = reinterpret_cast<int32_t*>(smem);      // [n + 1] prefix of live pages
  pdl_launch_dependents();
  // the call's own inputs may be read before the previous kernel has finished
  int sv[kPrefixPer];
#pragma unroll
  for (int e = 0; e < kPrefixPer; ++e) {
    const int i = tid * kPrefixPer + e;
    sv[e] = i < p.n ? __ldg(p.seq + i) : -1;
  }
  // everything below reads cache state: wait for the previous kernel
  pdl_wait();

  // ---- prefix of live pages over the call's sequences (per CTA; each
  //      thread takes kPrefixPer consecutive sequences of a pass) ----
  {
    int carry = 0;
    for (int base = 0; base < p.n; base += NT * kPrefixPer) {
      if (base > 0) {
#pragma unroll
        for (int e = 0; e < kPrefixPer; ++e) {
          const int i = base + tid * kPrefixPer + e;
          sv[e] = i < p.n ? __ldg(p.seq + i) : -1;
        }
      }
      int v[kPrefixPer];
#pragma unroll
      for (int e = 0; e < kPrefixPer; ++e) {
        const int i = base + tid * kPrefixPer + e;
        v[e] = 0;
        if (i < p.n) {
          const int s = sv[e];
          if (s >= 0 && s < p.max_seqs) v[e] = p.num_live[s];
          else if (blockIdx.x == 0) set_status(p.status, THINKV_ERR_INVALID);  // decoded as empty
        }
      }
      int tsum = 0;
#pragma unroll
      for (int e = 0; e < kPrefixPer; ++e) tsum += v[e];
      int x = tsum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xFFFFFFFFu, x, o);
        if (lane >= o) x += y;
      }
      if (lane == 31) wsum[warp] = x;
      __syncthreads();
      int before = carry, tot = 0;
      for (int w = 0; w < NW; ++w) {
        before += w < warp ? wsum[w] : 0;
        tot += wsum[w];
      }
      int run = before + x - tsum;
#pragma unroll
      for (int e = 0; e < kPrefixPer; ++e) {
        const int i = base + tid * kPrefixPer + e;
        if (i < p.n) P[i] = run;
        run += v[e];
      }
      carry += tot;
      __syncthreads();
    }
    if (tid == 0) P[p.n] = carry;
    __syncthreads();
  }
  write_empty_outputs(p, P, D);

  // ---- this CTA's share of the units, and this warp's part of it ----
  const int64_t T = (int64_t)P[p.n] * p.Hkv;
  const int64_t C = gridDim.x, cta = blockIdx.x;
  const int64_t U0c = cta * T / C, U1c = (cta + 1) * T / C, nuc = U1c - U0c;
  const int64_t U0 = U0c + warp * nuc / NW, U1 = U0c + (warp + 1) * nuc / NW;

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
  // the piece of this warp's first segment, when that segment started in an
  // earlier warp and ends in this one, goes to global memory (the ring is
  // busy then); a piece left at the end of the loop goes into the idle ring
  uint8_t* first_piece = p.wrec + ((int64_t)cta * NW + warp) * p.rb;
  // this warp's first and last segments, from the unit ranges (whatever the
  // loop below achieves, the merge duties stay the same)
  const int first_seg = U0 < U1 ? seg_of_unit(p, P, U0) : -1;
  const int last_seg = U0 < U1 ? seg_of_unit(p, P, U1 - 1) : -1;

  if (U0 < U1) {
    if (lane == 0) {
      for (int s2 = 0; s2 < p.nstage; ++s2) mbar_init(&bars[s2], 1);
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

    // every stage of the ring goes out at once: the first pages of all warps
    // are in flight together
    for (int s2 = 0; s2 < p.nstage && s2 < nu; ++s2) issue(cur, s2, s2);

    SegState<D, G> S;
    int seg = -1;
    int stage = 0;
    uint32_t parity = 0;
    bool failed = false;
    for (int k = 0; k < nu; ++k) {
      const int kk = k & 31;
      if (kk == 0 && k > 0) {
        cur = nxt;
        nxt = resolve_unit(p, P, U0 + k + 32 + lane, U1);
      }
      if (!mbar_wait_bounded(&bars[stage], parity)) {
        if (lane == 0) set_status(p.status, THINKV_ERR_TIMEOUT);
        // drain the copies still in flight (bounded), then stop computing;
        // the merges below still run (on stale pieces: the status says so)
        const int issued = min(nu, k + p.nstage);
        for (int k2 = k + 1; k2 < issued; ++k2)
          mbar_wait_bounded(&bars[k2 % p.nstage], (uint32_t)((k2 / p.nstage) & 1));
        failed = true;
        break;
      }
      const uint32_t cs = __shfl_sync(0xFFFFFFFFu, cur.cls_seg, kk);
      const int useg = (int)(cs & 0xFFFFFFu);
      uint8_t* blk = wsm + stage * p.stage_bytes;
      if (useg != seg) {
        if (seg >= 0) {
          // the previous segment ends inside this warp: whole here unless it
          // started before U0 (then it is this warp's first segment)
          int64_t Us, Ue;
          seg_range(p, P, seg / p.Hkv, seg % p.Hkv, &Us, &Ue);
          seg_end<D, G>(S, p, seg, tk, Us >= U0 ? nullptr : first_piece);
        }
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
    if (!failed) {
      int64_t Us, Ue;
      seg_range(p, P, seg / p.Hkv, seg % p.Hkv, &Us, &Ue);
      // the ring is idle now: every copy issued has landed
      seg_end<D, G>(S, p, seg, tk, (Us >= U0 && Ue <= U1) ? nullptr : wsm);
    }
  }
  if (lane == 0) s_last[warp] = last_seg;
  __syncthreads();

  // ---- merges: the last warp of this CTA that touches a split segment merges
  //      the warps' pieces; a segment spanning CTAs goes through the CTA records ----
  if (U0 >= U1) return;
  float* wbuf = pbuf;                              // the warp's 704-float merge scratch
  int* list = reinterpret_cast<int*>(pbuf) + 16;   // up to 160 piece owners
  for (int which = 0; which < 2; ++which) {
    const int S = which == 0 ? first_seg : last_seg;
    if (which == 0 && first_seg == last_seg) continue;   // one segment: handled as the last
    int64_t Us, Ue;
    seg_range(p, P, S / p.Hkv, S % p.Hkv, &Us, &Ue);
    if (Us >= U0 && Ue <= U1) continue;            // whole in this warp: already written
    // the last warp touching S merges: S ends in this warp, or this is the
    // CTA's last warp with units
    const int64_t wlast = share_of_unit(min(Ue, U1c) - 1 - U0c, nuc, NW);
    if (wlast != warp) continue;
    const int64_t wfirst = share_of_unit(max(Us, U0c) - U0c, nuc, NW);
    // the warps in [wfirst, warp] that hold units (shares can be empty when
    // the CTA has fewer units than warps)
    int npw = 0;
    for (int wj = (int)wfirst; wj <= warp; ++wj)
      if (U0c + (int64_t)wj * nuc / NW < U0c + (int64_t)(wj + 1) * nuc / NW) {
        if (lane == 0) list[npw] = wj;
        ++npw;
      }
    __syncwarp();
    auto warp_piece = [&](int j) -> const uint8_t* {
      const int wj = list[j];
      // a warp's piece of S sits in its ring if S was its last segment
      return s_last[wj] == S ? smem + p.plan_smem + wj * p.warp_smem
                             : p.wrec + ((int64_t)cta * NW + wj) * p.rb;
    };
    const bool in_cta = Us >= U0c && Ue <= U1c;
    if (in_cta) {
      merge_pieces<D, false>(p, S, npw, warp_piece, nullptr, wbuf);
      continue;
    }
    // the CTA's piece of S: slot 0 if S holds the CTA's first unit, else slot 1
    uint8_t* mine = p.crec + ((int64_t)cta * 2 + (Us <= U0c ? 0 : 1)) * p.rb;
    merge_pieces<D, false>(p, S, npw, warp_piece, mine, wbuf);
    __threadfence();
    __syncwarp();
    // the CTAs holding units of S (empty shares skipped)
    const int64_t ca = share_of_unit(Us, T, C), cb = share_of_unit(Ue - 1, T, C);
    int ncta = 0;
    for (int64_t c0 = ca; c0 <= cb; c0 += 32) {
      const int64_t cj = c0 + lane;
      const bool has = cj <= cb && cj * T / C < (cj + 1) * T / C;
      const unsigned bal = __ballot_sync(0xFFFFFFFFu, has);
      if (has) list[ncta + __popc(bal & ((1u << lane) - 1u))] = (int)cj;
      ncta += __popc(bal);
    }
    uint32_t old = 0;
    if (lane == 0) old = atomicInc(p.cnt + S, (uint32_t)ncta - 1u);   // wraps to 0 on the last arrival
    old = __shfl_sync(0xFFFFFFFFu, old, 0);
    if (old != (uint32_t)ncta - 1u) continue;
    __threadfence();                               // the other CTAs' records are visible now
    __syncwarp();
    auto cta_piece = [&](int j) -> const uint8_t* {
      const int64_t cj = list[j];
      const int64_t u0j = cj * T / C;
      return p.crec + (cj * 2 + (Us <= u0j ? 0 : 1)) * p.rb;
    };
    merge_pieces<D, true>(p, S, ncta, cta_piece, nullptr, wbuf);
  }
}

template <int D, int G>
cudaError_t launch_kernel(const DecodeParams& p, const DecodeLaunch& dl, cudaStream_t stream) {
  // raise the dynamic shared-memory limit of this instantiation once per
  // device (and again whenever a launch needs more); host threads that decode
  // at the same time serialise on the lock, so the recorded size never runs
  // ahead of the attribute actually set
  static std::mutex lock;
  static size_t configured[64] = {0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  {
    std::lock_guard<std::mutex> guard(lock);
    if (dl.smem_bytes > configured[dev]) {
      e = cudaFuncSetAttribute(decode_kernel<D, G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)dl.smem_bytes);
      if (e != cudaSuccess) return e;
      configured[dev] = dl.smem_bytes;
    }
  }
  return launch_pdl(decode_kernel<D, G>, dim3(dl.grid), dim3(dl.warps_per_cta * 32), dl.smem_bytes,
                    stream, p);
}

int plan_smem_bytes(int32_t n) { return ((n + 1) * 4 + 127) / 128 * 128; }

int64_t counters_bytes(const thinkv_layout& L, int32_t n) {
  return ((int64_t)n * L.num_kv_heads * 4 + 255) / 256 * 256;
}

}  // namespace

bool plan_decode_launch(const thinkv_layout& L, int32_t n_seqs, int32_t topk, int device,
                        DecodeLaunch* out) {
  const int D = L.head_dim, G = L.group_size;
  int64_t maxphb = 0;
  for (int c = 0; c < 3; ++c) {
    int64_t b = page_head_bytes(D, G, L.bits[c]);
    if (b > maxphb) maxphb = b;
  }
  const int Gq = L.num_q_heads / L.num_kv_heads;
  const int q_bytes = Gq * D * 2;
  const int stage_bytes = (int)((maxphb + 127) / 128 * 128) + (q_bytes + 127) / 128 * 128;
  const int topk_bytes = topk > 0 ? kTopkHdrBytes + Gq * kCandCap * 4 : 0;
  const int64_t rb = record_bytes(Gq, D, topk > 0 ? topk : 0);
  int optin = 0, sms = 0;
  if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, device) != cudaSuccess)
    return false;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device) != cudaSuccess) return false;
  // one CTA per SM: the stages take what the prefix, the per-warp scratch and
  // the kernel's static shared memory (under 1 KB) leave.  The most warps
  // that fit at least two stages each win (warps hide the page step's
  // latency; a deeper ring at fewer warps measured far slower), with as many
  // stages as fit; the ring must also hold the warp's last piece record
  const int64_t fixed = plan_smem_bytes(n_seqs) + 1024;
  int best_nw = 0, best_ns = 0;
  for (int nw = kDecWarps; nw >= 4 && best_nw == 0; --nw) {
    const int64_t per_warp = (optin - fixed) / nw - 64 - kPbufBytes - topk_bytes;
    int ns = per_warp > 0 ? (int)(per_warp / stage_bytes) : 0;
    if (ns > kMaxStages) ns = kMaxStages;
    if (ns < 2 || (int64_t)ns * stage_bytes < rb) continue;
    best_nw = nw;
    best_ns = ns;
  }
  if (best_nw == 0) return false;
  const int warp_smem = best_ns * stage_bytes + 64 + kPbufBytes + topk_bytes;
  const size_t smem = (size_t)plan_smem_bytes(n_seqs) + (size_t)best_nw * warp_smem;
  if (smem + 1024 > (size_t)optin) return false;
  // a segment's CTA list (merge scratch) holds up to 160 entries
  out->grid = sms < 160 ? sms : 160;
  out->warps_per_cta = best_nw;
  out->nstage = best_ns;
  out->stage_bytes = stage_bytes;
  out->smem_bytes = smem;
  out->warp_smem = warp_smem;
  out->pieces = (int64_t)out->grid * (best_nw + 2);
  return true;
}

size_t decode_workspace_bytes(const thinkv_layout& L, int32_t n_seqs, int32_t topk,
                              const DecodeLaunch& dl) {
  const int Gq = L.num_q_heads / L.num_kv_heads;
  // arrival counters, then the warps' and the CTAs' piece records
  return (size_t)counters_bytes(L, n_seqs) +
         (size_t)dl.pieces * (size_t)record_bytes(Gq, L.head_dim, topk > 0 ? topk : 0);
}

size_t decode_counter_bytes(const thinkv_layout& L, int32_t n_seqs) {
  return (size_t)counters_bytes(L, n_seqs);
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
    // the float formats take their own page steps (ternary is the 2-bit path)
    p.bits[c] = L.bits[c] + ((L.fmt[c] == 1 && L.bits[c] != 2) ? 256 : 0);
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
  p.topk = mass ? topk : 0;
  p.rb = (int32_t)record_bytes(p.Gq, D, p.topk);
  uint8_t* w = static_cast<uint8_t*>(ws);
  p.cnt = reinterpret_cast<uint32_t*>(w);
  w += counters_bytes(L, n);
  p.wrec = w;
  w += (int64_t)dl.grid * dl.warps_per_cta * p.rb;
  p.crec = w;
  p.nw = dl.warps_per_cta;
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
  if (D == 128 && G == 64) e = launch_kernel<128, 64>(p, dl, stream);
  else if (D == 128 && G == 32) e = launch_kernel<128, 32>(p, dl, stream);
  else if (D == 64 && G == 64) e = launch_kernel<64, 64>(p, dl, stream);
  else e = launch_kernel<64, 32>(p, dl, stream);
  return e;
}

}  // namespace thinkv
