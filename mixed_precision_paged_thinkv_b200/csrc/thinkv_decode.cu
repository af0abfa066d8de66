// thinkv_decode.cu -- decode attention over mixed-precision, slot-reusing pages.
//
// "ThinKV: Thought-Adaptive KV Cache Compression for Efficient Reasoning
// Models": the arXiv abstract's PagedAttention-based decode kernel, reading a
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
//   unpacks codes straight into mma.sync m16n8k16 operands (byte-permute
//   conversion to fp16 1024 + code), computes q.k for the whole GQA group at
//   once (tokens x heads), applies the per-group scale/zero in fp32, runs the
//   online softmax, forms p*scale (fp16, exponent-shifted) where the logits
//   are and moves it into the PV operand layout with register transposes
//   (movmatrix), and accumulates it times the centred V codes on the tensor
//   cores, with the zero terms summed in fp32.  A segment (sequence, kv-head)
//   that lies wholly in one warp is written out at once; otherwise each warp
//   writes one piece record (m, l, o, top-k candidates) per segment it touched.
//
//   combine kernel (launched right behind, programmatic dependent launch): one
//   CTA per segment left in several pieces merges the records with the
//   log-sum-exp rule -- a thread per quad of each head's output row, a warp per
//   head sorting and merging the pieces' top-k candidates -- and writes fp16 O
//   and the top-k mass.
#include <cuda_fp16.h>
#include <limits.h>
#include <mutex>
#include <stdint.h>

#include "thinkv_common.cuh"
#include "thinkv_internal.h"

namespace thinkv {

namespace {

// Split CTA shape per head dim: warps per CTA, and CTAs per SM the kernel is
// built for (its register cap follows).  A d = 128 page step wants up to 168
// registers: three 4-warp CTAs.  A d = 64 one fits in 128: two 8-warp CTAs,
// 16 warps per SM, ran 6-10 % faster than 12 warps at 168.
template <int D>
struct SplitShape {
  static constexpr int warps = D == 64 ? 8 : 4;
  static constexpr int ctas = D == 64 ? 2 : 3;
  static constexpr int threads = warps * 32;
  static constexpr int regs = 65536 / (threads * ctas) / 8 * 8;   // 128 | 168
};
// per-warp scratch: the segment's Q fragments, lane-contiguous (the B
// operands of the QK products)
constexpr int kQfragOff = 0;
__host__ __device__ constexpr int pbuf_bytes(int D) { return D / 16 * 32 * 8; }  // k-steps x lanes x 8 B
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
  void* rec;         // piece records of split segments (index warp + segment)
  int32_t* pref;      // [n + 1] prefix of live pages over the call's sequences
  int64_t split_warps;  // warps of the split kernel's grid
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
//   then (with the top-k statistic) 4*Gq*kCandCap bytes: per head, the
//                           piece's candidate logits -- a superset of its topk
//                           largest -- unsorted, -inf padded
__host__ __device__ inline int64_t record_bytes(int Gq, int D, int topk) {
  return 64 + 4LL * Gq * D + (topk > 0 ? 4LL * Gq * kCandCap : 0);
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

// The warp of the stream-K split (warp w holds units [w*T/W, (w+1)*T/W))
// that holds unit u.
__device__ inline int64_t warp_of_unit(int64_t u, int64_t T, int64_t W) {
  return ((u + 1) * W - 1) / T;
}

// Ends the warp's work on segment seg = i * Hkv + h.  If the whole segment
// was in this warp (Us >= U0 and Ue <= U1) its O rows and top-k mass are
// written at once; otherwise the warp's piece record goes to rec[w + seg]
// for the merge.
template <int D, int G, bool TOPK>
__device__ inline void seg_end(SegState<D, G>& S, const DecodeParams& p, int64_t w, int seg,
                               const TopkCtx& tk, bool whole) {
  constexpr int NG = SegState<D, G>::NG, MT = SegState<D, G>::MT;
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int i = seg / p.Hkv, h = seg - (seg / p.Hkv) * p.Hkv;
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
  const int64_t rb = record_bytes(Gq, D, tk.topk);
  uint8_t* rec = reinterpret_cast<uint8_t*>(p.rec) + (w + seg) * rb;
  float* po = reinterpret_cast<float*>(rec + 64);
  const float li0 = whole ? 1.f / S.lp[0] : 1.f, li1 = whole ? 1.f / S.lp[1] : 1.f;
  if (!whole && g == 0) {
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const int hd = 2 * t + c;
      if (hd < Gq) reinterpret_cast<float2*>(rec)[hd] = make_float2(S.m[c], S.lp[c]);
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
  if (TOPK && tk.topk > 0) {
    if (!whole) {
      // a piece hands its candidate buffers over as they are (each a superset
      // of its head's topk largest; -inf past the count): the combine sorts
      // them, a warp per head
      float* tl = reinterpret_cast<float*>(rec + 64 + 4 * Gq * D);
      for (int hd = 0; hd < Gq; ++hd) {
        const int n = tk.cnt[hd];
        float4 v = *reinterpret_cast<const float4*>(tk.cand + hd * kCandCap + 4 * lane);
        if (4 * lane + 0 >= n) v.x = -INFINITY;
        if (4 * lane + 1 >= n) v.y = -INFINITY;
        if (4 * lane + 2 >= n) v.z = -INFINITY;
        if (4 * lane + 3 >= n) v.w = -INFINITY;
        *reinterpret_cast<float4*>(tl + hd * kCandCap + 4 * lane) = v;
      }
    } else {
      const bool all = p.live_count[p.seq[i]] <= tk.topk;
      for (int hd = 0; hd < Gq; ++hd) {
        float sum = 0.f;
        if (!all) {
          if (tk.topk <= 32 && tk.cnt[hd] > 64) cand_prune(tk, hd);   // then the 64-wide sort
          if (tk.cnt[hd] > 0) cand_compact(tk, hd);      // sorted, the k largest kept
          const int n = tk.cnt[hd];
          const float m = __shfl_sync(0xFFFFFFFFu, (hd & 1) ? S.m[1] : S.m[0], hd >> 1);
          for (int j = lane; j < n; j += 32) sum += exp2_approx(tk.cand[hd * kCandCap + j] - m);
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
        }
        const float l = __shfl_sync(0xFFFFFFFFu, (hd & 1) ? S.lp[1] : S.lp[0], hd >> 1);
        if (lane == 0) p.mass[(int64_t)i * p.Hq + h * Gq + hd] = all ? 1.f : sum / l;
      }
    }
  }
  __syncwarp();
}

// Transpose of an 8x8 matrix of 16-bit elements held one register per lane
// (lane 4r + c holds row r, columns 2c and 2c + 1): afterwards the lane holds
// row r of the transpose, i.e. column r of the original.
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t a) {
  uint32_t d;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(d) : "r"(a));
  return d;
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
template <int D, int G, int B, int F, bool TOPK>
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
      // two accumulator chains (even and odd k-steps) halve the dependent
      // MMA latency of a group
      float c2[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
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
        mma_16816(c2[s & 1], a, qb.x, qb.y);
      }
      const float c[4] = {c2[0][0] + c2[1][0], c2[0][1] + c2[1][1], c2[0][2] + c2[1][2],
                          c2[0][3] + c2[1][3]};
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
  if (TOPK && tk.topk > 0) {
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

  // V scales of this lane's tokens g and g + 8, per group (the rows the zero term reads)
  float s0[NG], s1[NG];
#pragma unroll
  for (int gr = 0; gr < NG; ++gr) {
    if constexpr (B == 16) {
      s0[gr] = s1[gr] = 1.f;
    } else {
      const uint32_t p0 = vpar[gr * 16 + g], p1 = vpar[gr * 16 + g + 8];
      const float2 sz0 = __half22float2(*reinterpret_cast<const __half2*>(&p0));
      const float2 sz1 = __half22float2(*reinterpret_cast<const __half2*>(&p1));
      s0[gr] = sz0.x;
      s1[gr] = sz1.x;
      constexpr float voff = F == 1 ? 0.f : (float)(1 << (B - 1));
      const float zv0 = live0 ? fmaf(voff, sz0.x, sz0.y) : 0.f;
      const float zv1 = live1 ? fmaf(voff, sz1.x, sz1.y) : 0.f;
      S.z[gr][0] = fmaf(S.z[gr][0], a0, fmaf(pr[0], zv0, pr[2] * zv1));
      S.z[gr][1] = fmaf(S.z[gr][1], a1, fmaf(pr[1], zv0, pr[3] * zv1));
    }
  }

  // ---------------- PV operands W = p * s_V * 2^sigma (one sigma per segment),
  //   formed where the logits are (tokens g, g+8; heads 2t, 2t+1), packed to
  //   fp16 and moved to the B-operand layout (tokens 2t, 2t+1, 2t+8, 2t+9;
  //   head g) by an 8x8 register transpose per token half ----------------
  // dead slots of the V operand (float codes, raw fp16): zeroed in the A operand
  const uint32_t tmask = mask >> (2 * t);
  const uint32_t dm0 = ((tmask & 1u) ? 0xFFFFu : 0u) | ((tmask & 2u) ? 0xFFFF0000u : 0u);
  const uint32_t dm1 = ((tmask & 0x100u) ? 0xFFFFu : 0u) | ((tmask & 0x200u) ? 0xFFFF0000u : 0u);
  float f = S.sigma == kSigmaInit ? 0.f : pow2i(S.sigma);
  float wv[NG][4];
  float wmax = 0.f;
#pragma unroll
  for (int gr = 0; gr < NG; ++gr) {
    wv[gr][0] = pr[0] * f * s0[gr];
    wv[gr][1] = pr[1] * f * s0[gr];
    wv[gr][2] = pr[2] * f * s1[gr];
    wv[gr][3] = pr[3] * f * s1[gr];
    wmax = live0 ? fmaxf(wmax, fmaxf(wv[gr][0], wv[gr][1])) : wmax;
    wmax = live1 ? fmaxf(wmax, fmaxf(wv[gr][2], wv[gr][3])) : wmax;
  }
  float fac = 1.f;
  // slow path: first page of the segment, or a scale large enough to overflow fp16
  if (__any_sync(0xFFFFFFFFu, S.sigma == kSigmaInit || !(wmax < 32768.f))) {
    int e5 = 1;
#pragma unroll
    for (int gr = 0; gr < NG; ++gr) {
      const int ef0 = (__float_as_int(s0[gr]) >> 23) - 112;   // fp16 exponent field
      const int ef1 = (__float_as_int(s1[gr]) >> 23) - 112;
      e5 = live0 ? max(e5, ef0) : e5;
      e5 = live1 ? max(e5, ef1) : e5;
    }
    // over the page's 16 tokens: the lanes of other g hold the other tokens
    e5 = max(e5, __shfl_xor_sync(0xFFFFFFFFu, e5, 4));
    e5 = max(e5, __shfl_xor_sync(0xFFFFFFFFu, e5, 8));
    e5 = max(e5, __shfl_xor_sync(0xFFFFFFFFu, e5, 16));
    const int sp = 29 - e5;             // s * 2^sp < 2^15 for every live scale of the page
    if (sp < S.sigma) {
      if (S.sigma != kSigmaInit) fac = pow2i(sp - S.sigma);
      S.sigma = sp;
    }
    f = pow2i(S.sigma);
#pragma unroll
    for (int gr = 0; gr < NG; ++gr) {
      wv[gr][0] = pr[0] * f * s0[gr];
      wv[gr][1] = pr[1] * f * s0[gr];
      wv[gr][2] = pr[2] * f * s1[gr];
      wv[gr][3] = pr[3] * f * s1[gr];
    }
  }
  uint32_t wf[NG][2];
#pragma unroll
  for (int gr = 0; gr < NG; ++gr) {
    // dead tokens: p is 0, but their stale scales may not be finite
    const uint32_t lo = live0 ? pack_half2_rn(wv[gr][0], wv[gr][1]) : 0u;   // token g
    const uint32_t hi = live1 ? pack_half2_rn(wv[gr][2], wv[gr][3]) : 0u;   // token g + 8
    wf[gr][0] = movmatrix_trans(lo);    // head g: tokens 2t, 2t+1
    wf[gr][1] = movmatrix_trans(hi);    // head g: tokens 2t+8, 2t+9
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
template <int D, int G, bool TOPK>
__device__ inline void page_dispatch(SegState<D, G>& S, const uint8_t* blk, int bits, uint32_t mask,
                                     float scale_log2, float* pbuf, const TopkCtx& tk, int Gq) {
  switch (bits) {
    case 256 + 8: page_step<D, G, 8, 1, TOPK>(S, blk, mask, scale_log2, pbuf, tk, Gq); break;
    case 256 + 4: page_step<D, G, 4, 1, TOPK>(S, blk, mask, scale_log2, pbuf, tk, Gq); break;
    case 8: page_step<D, G, 8, 0, TOPK>(S, blk, mask, scale_log2, pbuf, tk, Gq); break;
    case 4: page_step<D, G, 4, 0, TOPK>(S, blk, mask, scale_log2, pbuf, tk, Gq); break;
    case 2: page_step<D, G, 2, 0, TOPK>(S, blk, mask, scale_log2, pbuf, tk, Gq); break;
    default: page_step<D, G, 16, 0, TOPK>(S, blk, mask, scale_log2, pbuf, tk, Gq); break;
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
  const int64_t row = (int64_t)P[p.n + 1 + i] * p.max_blocks;   // the sequence id, cached
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

template <int D, int G, bool TOPK>
__global__ void __launch_bounds__(SplitShape<D>::threads, SplitShape<D>::ctas)
    decode_split_kernel(DecodeParams p) {
  constexpr int kDecWarps = SplitShape<D>::warps, kDecThreads = SplitShape<D>::threads;
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int32_t* P = reinterpret_cast<int32_t*>(smem);      // [n + 1] prefix of live pages
  int32_t* Sq = P + (p.n + 1);                         // [n] the call's sequence ids
  pdl_launch_dependents();
  // the call's own inputs may be read before the previous kernel has finished
  for (int i = tid; i < p.n; i += kDecThreads) Sq[i] = p.seq[i];
  // everything below reads cache state: wait for the previous kernel
  pdl_wait();
  __syncthreads();

  // ---- prefix of live pages over the call's sequences (per CTA) ----
  {
    __shared__ int wsum[kDecWarps];
    int carry = 0;
    for (int base = 0; base < p.n; base += kDecThreads) {
      const int i = base + tid;
      int v = 0;
      if (i < p.n) {
        const int s = Sq[i];
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
  if (blockIdx.x == 0)
    for (int x = tid; x <= p.n; x += kDecThreads) p.pref[x] = P[x];   // for the combine
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
    uint8_t* tb = wsm + p.nstage * p.stage_bytes + 64 + pbuf_bytes(D);
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
  bool failed = false;
  for (int k = 0; k < nu; ++k) {
    const int kk = k & 31;
    if (kk == 0 && k > 0) {
      cur = nxt;
      nxt = resolve_unit(p, P, U0 + k + 32 + lane, U1);
    }
    if (!mbar_wait_bounded(&bars[stage], parity)) {
      if (lane == 0) set_status(p.status, THINKV_ERR_TIMEOUT);
      // drain the copies still in flight (bounded), then stop
      const int issued = k == 0 ? 1 : min(nu, k + p.nstage);
      for (int k2 = k + 1; k2 < issued; ++k2)
        mbar_wait_bounded(&bars[k2 % p.nstage], (uint32_t)((k2 / p.nstage) & 1));
      failed = true;
      break;
    }
    if (k == 0)
      for (int s2 = 1; s2 < p.nstage && s2 < nu; ++s2) issue(cur, s2, s2);
    const uint32_t cs = __shfl_sync(0xFFFFFFFFu, cur.cls_seg, kk);
    const int useg = (int)(cs & 0xFFFFFFu);
    uint8_t* blk = wsm + stage * p.stage_bytes;
    if (useg != seg) {
      if (seg >= 0) {
        int64_t Us, Ue;
        seg_range(p, P, seg / p.Hkv, seg % p.Hkv, &Us, &Ue);
        seg_end<D, G, TOPK>(S, p, w, seg, tk, Us >= U0 && Ue <= U1);
      }
      seg = useg;
      seg_begin<D, G>(S, p, reinterpret_cast<const uint16_t*>(blk + p.q_off),
                      reinterpret_cast<uint2*>(reinterpret_cast<uint8_t*>(pbuf) + kQfragOff), tk);
      __syncwarp();
    }
    const uint32_t mask = __shfl_sync(0xFFFFFFFFu, cur.mask, kk);
    page_dispatch<D, G, TOPK>(S, blk, p.bits[cs >> 24], mask & 0xFFFFu, p.scale_log2, pbuf, tk, p.Gq);
    __syncwarp();
    // refill this stage with unit k + nstage (from this batch of 32 or the next)
    const int kn = k + p.nstage;
    if (kn < nu) issue(((kn >> 5) == (k >> 5)) ? cur : nxt, kn, stage);
    if (++stage == p.nstage) {
      stage = 0;
      parity ^= 1u;
    }
  }
  if (failed || seg < 0) return;
  {
    int64_t Us, Ue;
    seg_range(p, P, seg / p.Hkv, seg % p.Hkv, &Us, &Ue);
    seg_end<D, G, TOPK>(S, p, w, seg, tk, Us >= U0 && Ue <= U1);
  }
}


// ---------------------------------------------------------------------------
// split combine: one CTA per (sequence, kv-head) segment that the split
// kernel left in more than one piece
// ---------------------------------------------------------------------------
constexpr int kCombineThreads = 256;            // the most a combine CTA takes
constexpr int kCombinePieces = 128;             // pieces per round of the weight table

// Merges the segment's piece records with the log-sum-exp rule: thread t <
// Gq * D/4 owns one quad of one head's output row; warp r < Gq then sorts each
// piece's top-k candidates for head r and merges their largest into a running
// list (bitonic networks, the next piece's candidates loaded while the current
// ones are sorted) for the top-k mass.
template <int D, bool TOPK>
__global__ void __launch_bounds__(kCombineThreads, TOPK ? 4 : 3) decode_combine_kernel(DecodeParams p) {
  constexpr int QD = D / 4;
  __shared__ float sM[8], sL[8];
  __shared__ int sMk[8];
  __shared__ float cwt[kCombinePieces * 8], lt[kCombinePieces * 8];
  pdl_launch_dependents();
  pdl_wait();                                   // records and prefix come from the split kernel
  const int seg = blockIdx.x;
  const int i = seg / p.Hkv, h = seg - (seg / p.Hkv) * p.Hkv;
  const int nl = p.pref[i + 1] - p.pref[i];
  if (nl == 0) return;                          // written by the split kernel
  const int64_t T = (int64_t)p.pref[p.n] * p.Hkv, W = p.split_warps;
  const int64_t Us = (int64_t)p.pref[i] * p.Hkv + (int64_t)h * nl, Ue = Us + nl;
  const int64_t w0 = warp_of_unit(Us, T, W), w1 = warp_of_unit(Ue - 1, T, W);
  const bool by_unit = T <= W;                  // one unit per warp
  const int np = (int)(by_unit ? nl : w1 - w0 + 1);
  if (np <= 1) return;                          // finished inside one split warp
  const int Gq = p.Gq, k = p.topk;
  // the top-k warps' live count, requested now and used after the merge
  const int live_i = (p.mass && threadIdx.x < 32 * Gq) ? p.live_count[p.seq[i]] : 0;
  const int64_t rb = record_bytes(Gq, D, k);
  const uint8_t* recs = reinterpret_cast<const uint8_t*>(p.rec);
  auto rec = [&](int j) -> const uint8_t* {
    const int64_t pc = (by_unit ? warp_of_unit(Us + j, T, W) : w0 + j) + seg;
    return recs + pc * rb;
  };
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // pieces whose quads are requested up front (fewer with top-k, whose CTAs
  // are built to fit four to an SM)
  constexpr int kCombinePre = TOPK ? 4 : 8;

  // ---- per piece and head: the weight 2^(m - M) (M the head's max), and L ----
  // (m, l) pairs are read once, lane-parallel; a table of weights in shared
  // memory then lets every output thread stream its quads with many loads in
  // flight.  Segments with more pieces than the table holds go in rounds.
  float* wt = cwt;                                // [kCombinePieces][8]
  // a float's order-preserving int key (negative floats: magnitude bits
  // flipped); the map is its own inverse
  auto okey = [](int b) { return b >= 0 ? b : b ^ 0x7FFFFFFF; };
  const int r_o = tid / QD, q_o = tid - (tid / QD) * QD;
  const bool out_thread = tid < Gq * QD;
  auto quad = [&](int j) {
    return __ldcg(reinterpret_cast<const float4*>(rec(j) + 64) + r_o * QD + q_o);
  };
  auto pair_ml = [&](int x) {
    const int j = x / Gq, r = x - j * Gq;
    return __ldcg(reinterpret_cast<const float2*>(rec(j)) + r);
  };
  // the first pieces' quads and (m, l) pairs do not depend on the weights:
  // all of them are requested at once
  float4 ov[kCombinePre];
#pragma unroll
  for (int j = 0; j < kCombinePre; ++j)
    ov[j] = (out_thread && j < np) ? quad(j) : make_float4(0.f, 0.f, 0.f, 0.f);
  const float2 ml0 = tid < np * Gq ? pair_ml(tid) : make_float2(-INFINITY, 0.f);
  if (tid < 8) { sMk[tid] = INT_MIN; sL[tid] = 0.f; }
  __syncthreads();
  for (int x = tid; x < np * Gq; x += (int)blockDim.x) {
    const float m = x == tid ? ml0.x : pair_ml(x).x;
    atomicMax(&sMk[x - (x / Gq) * Gq], okey(__float_as_int(m)));
  }
  __syncthreads();
  if (tid < 8) sM[tid] = __int_as_float(okey(sMk[tid]));
  __syncthreads();
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int j0 = 0; j0 < np; j0 += kCombinePieces) {
    const int cnt = min(kCombinePieces, np - j0);
    for (int x = tid; x < cnt * Gq; x += (int)blockDim.x) {
      const int j = x / Gq, r = x - j * Gq;
      const float2 ml = (j0 == 0 && x == tid) ? ml0 : pair_ml(j0 * Gq + x);
      const float wgt = exp2_approx(ml.x - sM[r]);
      wt[j * 8 + r] = wgt;
      lt[j * 8 + r] = wgt * ml.y;
    }
    __syncthreads();
    if (warp < Gq) {                              // L, summed in a fixed order
      float l = 0.f;
      for (int j = lane; j < cnt; j += 32) l += lt[j * 8 + warp];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xFFFFFFFFu, l, o);
      if (lane == 0) sL[warp] += l;
    }
    if (out_thread) {
      int jstart = 0;
      if (j0 == 0) {
#pragma unroll
        for (int j = 0; j < kCombinePre; ++j) {
          const float wgt = j < cnt ? wt[j * 8 + r_o] : 0.f;
          acc.x = fmaf(wgt, ov[j].x, acc.x);
          acc.y = fmaf(wgt, ov[j].y, acc.y);
          acc.z = fmaf(wgt, ov[j].z, acc.z);
          acc.w = fmaf(wgt, ov[j].w, acc.w);
        }
        jstart = kCombinePre;
      }
#pragma unroll 8
      for (int j = jstart; j < cnt; ++j) {
        const float4 v = quad(j0 + j);
        const float wgt = wt[j * 8 + r_o];
        acc.x = fmaf(wgt, v.x, acc.x);
        acc.y = fmaf(wgt, v.y, acc.y);
        acc.z = fmaf(wgt, v.z, acc.z);
        acc.w = fmaf(wgt, v.w, acc.w);
      }
    }
    __syncthreads();                              // the table is refilled by the next round
  }
  if (tid < Gq * QD) {
    const float inv = 1.f / sL[r_o];
    const uint32_t lo = (uint32_t)__half_as_ushort(__float2half_rn(acc.x * inv)) |
                        ((uint32_t)__half_as_ushort(__float2half_rn(acc.y * inv)) << 16);
    const uint32_t hi = (uint32_t)__half_as_ushort(__float2half_rn(acc.z * inv)) |
                        ((uint32_t)__half_as_ushort(__float2half_rn(acc.w * inv)) << 16);
    const int64_t row = (int64_t)i * p.Hq + h * Gq + r_o;
    reinterpret_cast<uint2*>(p.out + row * D)[q_o] = make_uint2(lo, hi);
  }
  if (!p.mass) return;
  if (warp >= Gq) return;
  const int r = warp;
  const int64_t mrow = (int64_t)i * p.Hq + h * Gq + r;
  if (live_i <= k) {
    if (lane == 0) p.mass[mrow] = 1.f;
    return;
  }
  // The running list holds the 64 largest candidates so far, descending, in
  // elements 0..63 (lane * 4 + e); its k-th element is exact, the rest of it
  // need not be.  A piece's candidates at or below that k-th value cannot
  // enter the top k (a tie leaves the sum unchanged) and are dropped.  Up to
  // 32 survivors are gathered one per lane, sorted (32-wide network) and put
  // rising in elements 96..127 (-inf in 64..95); more are sorted whole, their
  // 64 largest rising in elements 64..127.  Either way, with the running list
  // in 0..63 that is a bitonic sequence, which one merge puts in order.
  float tv[4], nx[4];
  auto load_list = [&](int j, float (&x)[4]) {
    const float4 v = __ldcg(reinterpret_cast<const float4*>(rec(j) + 64 + 4 * Gq * D) +
                            r * (kCandCap / 4) + lane);
    x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
  };
  float* ys = cwt + warp * 32;                    // gather slots (the weight table is free now)
  unsigned below;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(below));
  // the survivors (at most 32) of this lane's candidates x, one per lane
  // (-inf past the c-th), in descending order
  auto gather_sorted = [&](const float (&x)[4], const unsigned (&b)[4], float th, int c) {
    int at = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (x[e] > th) ys[at + __popc(b[e] & below)] = x[e];
      at += __popc(b[e]);
    }
    __syncwarp();
    const float y = lane < c ? ys[lane] : -INFINITY;
    __syncwarp();                                 // the slots are rewritten by the next piece
    return bitonic32_desc(y);
  };
  const float M = sM[r];
  if (k <= 32) {
    // k <= 32: the running list is the 32 largest so far, one per lane,
    // descending (lane 0 the largest); its k-th element is the threshold
    float rv = -INFINITY;
    load_list(0, nx);
    for (int j = 0; j < np; ++j) {
      float x[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) x[e] = nx[e];
      if (j + 1 < np) load_list(j + 1, nx);
      const float th = __shfl_sync(0xFFFFFFFFu, rv, k - 1);
      unsigned b[4];
      int c = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        b[e] = __ballot_sync(0xFFFFFFFFu, x[e] > th);
        c += __popc(b[e]);
      }
      if (c == 0) continue;
      float y;
      if (c <= 32) {
        y = gather_sorted(x, b, th, c);
      } else {
        float v[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) v[e] = -x[e];
        bitonic128_desc(v);                       // descending of -x: ascending of x
        // the lane-th largest is element 127 - lane: lane 31 - lane/4, slot 3 - lane%4
        const int sl = 31 - (lane >> 2), se = 3 - (lane & 3);
        const float t0 = __shfl_sync(0xFFFFFFFFu, v[0], sl), t1 = __shfl_sync(0xFFFFFFFFu, v[1], sl);
        const float t2 = __shfl_sync(0xFFFFFFFFu, v[2], sl), t3 = __shfl_sync(0xFFFFFFFFu, v[3], sl);
        y = -(se == 0 ? t0 : (se == 1 ? t1 : (se == 2 ? t2 : t3)));
      }
      // the 32 largest of two descending lists: each element against the
      // other list's mirror element; the maxima form a bitonic sequence
      float z = fmaxf(rv, __shfl_sync(0xFFFFFFFFu, y, 31 - lane));
#pragma unroll
      for (int stride = 16; stride > 0; stride >>= 1) {
        const float o = __shfl_xor_sync(0xFFFFFFFFu, z, stride);
        z = (lane & stride) == 0 ? fmaxf(z, o) : fminf(z, o);
      }
      rv = z;
    }
    float sum = lane < k ? exp2_approx(rv - M) : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
    if (lane == 0) p.mass[mrow] = sum / sL[r];
    return;
  }
  const int ke = (k - 1) & 3, kl = (k - 1) >> 2;  // the k-th element: lane kl, slot ke
#pragma unroll
  for (int e = 0; e < 4; ++e) tv[e] = -INFINITY;
  load_list(0, nx);
  for (int j = 0; j < np; ++j) {
    float x[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) x[e] = nx[e];
    if (j + 1 < np) load_list(j + 1, nx);
    const float kv = ke == 0 ? tv[0] : (ke == 1 ? tv[1] : (ke == 2 ? tv[2] : tv[3]));
    const float th = __shfl_sync(0xFFFFFFFFu, kv, kl);
    unsigned b[4];
    int c = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      b[e] = __ballot_sync(0xFFFFFFFFu, x[e] > th);
      c += __popc(b[e]);
    }
    if (c == 0) continue;
    float v[4];
    if (c <= 32) {
      const float y = gather_sorted(x, b, th, c);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int m = (lane - 24) * 4 + e;        // rank in the rising run of lanes 24..31
        const float ya = __shfl_sync(0xFFFFFFFFu, y, (31 - m) & 31);
        v[e] = lane < 16 ? tv[e] : (lane >= 24 ? ya : -INFINITY);
      }
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e) v[e] = -x[e];
      bitonic128_desc(v);                         // descending of -x: ascending of x
#pragma unroll
      for (int e = 0; e < 4; ++e) v[e] = (lane * 4 + e < 64) ? tv[e] : -v[e];
    }
    bitonic128_merge_desc(v);
#pragma unroll
    for (int e = 0; e < 4; ++e) tv[e] = v[e];
  }
  float sum = 0.f;
#pragma unroll
  for (int e = 0; e < 4; ++e)
    if (lane * 4 + e < k) sum += exp2_approx(tv[e] - M);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
  if (lane == 0) p.mass[mrow] = sum / sL[r];
}

template <int D, int G, bool TOPK>
cudaError_t launch_split_t(const DecodeParams& p, const DecodeLaunch& dl, cudaStream_t stream) {
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
      e = cudaFuncSetAttribute(decode_split_kernel<D, G, TOPK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)dl.smem_bytes);
      if (e != cudaSuccess) return e;
      configured[dev] = dl.smem_bytes;
    }
  }
  e = launch_pdl(decode_split_kernel<D, G, TOPK>, dim3(dl.grid), dim3(SplitShape<D>::threads), dl.smem_bytes,
                 stream, p);
  if (e != cudaSuccess) return e;
  // the combine: one CTA per segment (most return at once), as many threads as
  // the segment's output quads (Gq * D/4), and a warp per head at least (the
  // per-head sums, the top-k merges)
  const int qt = (p.Gq * (D / 4) + 31) / 32 * 32;
  const int ct = qt > 32 * p.Gq ? qt : 32 * p.Gq;
  return launch_pdl(decode_combine_kernel<D, TOPK>, dim3((unsigned)(p.n * p.Hkv)),
                    dim3(ct < kCombineThreads ? ct : kCombineThreads), 0, stream, p);
}

// the top-k candidate code is compiled only into the instantiation that uses it
template <int D, int G>
cudaError_t launch_split(const DecodeParams& p, const DecodeLaunch& dl, cudaStream_t stream) {
  return p.topk > 0 ? launch_split_t<D, G, true>(p, dl, stream) : launch_split_t<D, G, false>(p, dl, stream);
}

int plan_smem_bytes(int32_t n) { return ((2 * n + 1) * 4 + 127) / 128 * 128; }

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
  const int Gq = L.num_q_heads / L.num_kv_heads;
  const int topk_bytes = topk > 0 ? kTopkHdrBytes + Gq * kCandCap * 4 : 0;
  const int warps = D == 64 ? SplitShape<64>::warps : SplitShape<128>::warps;
  const int ctas = D == 64 ? SplitShape<64>::ctas : SplitShape<128>::ctas;
  const int regs = D == 64 ? SplitShape<64>::regs : SplitShape<128>::regs;
  int smem_per_sm = 0;
  if (cudaDeviceGetAttribute(&smem_per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, device) !=
      cudaSuccess)
    return false;
  // page-head stages and top-k buffers: ~15 KB per warp, less where the CTA
  // shape leaves less (1 KB of each CTA reserved); a deeper ring measured no
  // faster: warps, not ring depth, hide the page step
  int budget = (smem_per_sm / ctas - 1024 - plan_smem_bytes(n_seqs)) / warps - 64 - pbuf_bytes(D);
  if (budget > 15360) budget = 15360;
  int nstage = (budget - topk_bytes) / stage_bytes;
  if (nstage < 2) nstage = 2;
  if (nstage > kMaxStages) nstage = kMaxStages;
  const int warp_smem = nstage * stage_bytes + 64 + pbuf_bytes(D) + topk_bytes;
  const size_t smem = (size_t)plan_smem_bytes(n_seqs) + (size_t)warps * warp_smem;
  int optin = 0;
  if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, device) != cudaSuccess)
    return false;
  if (smem + 1024 > (size_t)optin) return false;
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device) != cudaSuccess) return false;
  // CTAs per SM: limited by shared memory (1 KB reserved per CTA) and by registers
  int per_sm = smem_per_sm / (int)(smem + 1024);
  int regs_per_sm = 0;
  if (cudaDeviceGetAttribute(&regs_per_sm, cudaDevAttrMaxRegistersPerMultiprocessor, device) !=
      cudaSuccess)
    return false;
  const int by_regs = regs_per_sm / (regs * warps * 32);
  if (per_sm > by_regs) per_sm = by_regs;
  if (per_sm > 16) per_sm = 16;
  if (per_sm < 1) per_sm = 1;
  out->grid = sms * per_sm;
  out->warps_per_cta = warps;
  out->nstage = nstage;
  out->stage_bytes = stage_bytes;
  out->smem_bytes = smem;
  out->warp_smem = warp_smem;
  out->pieces = (int64_t)out->grid * warps + (int64_t)n_seqs * L.num_kv_heads;

  return true;
}

size_t decode_workspace_bytes(const thinkv_layout& L, int32_t n_seqs, int32_t topk,
                              const DecodeLaunch& dl) {
  const int Gq = L.num_q_heads / L.num_kv_heads;
  // the prefix of live pages, then one record per (split warp, segment)
  const size_t head = (size_t)(n_seqs + 1 > n_seqs * L.num_kv_heads ? n_seqs + 1
                                                                     : n_seqs * L.num_kv_heads);
  size_t b = (head * 4 + 255) / 256 * 256;
  b += (size_t)dl.pieces * (size_t)record_bytes(Gq, L.head_dim, topk > 0 ? topk : 0);
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
  uint8_t* w = static_cast<uint8_t*>(ws);
  p.pref = reinterpret_cast<int32_t*>(w);
  {
    const size_t head = (size_t)(n + 1 > n * L.num_kv_heads ? n + 1 : n * L.num_kv_heads);
    w += (head * 4 + 255) / 256 * 256;
  }
  p.topk = mass ? topk : 0;
  p.rec = w;
  p.split_warps = (int64_t)dl.grid * dl.warps_per_cta;
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
