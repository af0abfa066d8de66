// thinkv_api.cu -- the extern "C" entry points of libthinkv.so (see include/thinkv.h).
//
// Host-side argument checks, buffer-size arithmetic, cache reset and status
// handling; every operation itself runs in the kernels of thinkv_append.cu,
// thinkv_evict.cu and thinkv_decode.cu.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "thinkv.h"
#include "thinkv_common.cuh"
#include "thinkv_internal.h"

using namespace thinkv;

namespace {

bool layout_ok(const thinkv_layout* L) {
  if (!L) return false;
  if (L->page_size != kPage) return false;
  if (L->num_kv_heads <= 0 || L->num_q_heads <= 0) return false;
  if (L->num_q_heads % L->num_kv_heads) return false;
  if (L->num_q_heads / L->num_kv_heads > 8) return false;
  if (L->head_dim != 64 && L->head_dim != 128) return false;
  if (L->group_size != 32 && L->group_size != 64) return false;
  if (L->head_dim % L->group_size) return false;
  for (int c = 0; c < 3; ++c) {
    const int b = L->bits[c];
    if (b != 2 && b != 4 && b != 8 && b != 16) return false;
    if (L->pool_pages[c] < 0 || L->pool_pages[c] >= (1 << 27)) return false;
    if (L->fmt[c] != THINKV_FMT_INT && !(L->fmt[c] == THINKV_FMT_FLOAT && b != 16)) return false;
  }
  if (L->max_seqs < 1 || L->max_seqs > 65536) return false;
  if (L->max_blocks_per_seq < 1 || L->max_blocks_per_seq > (1 << 21)) return false;
  if (L->num_kv_heads > 256) return false;
  return true;
}

}  // namespace

namespace thinkv {

bool cache_ok(const thinkv_cache* C) {
  if (!C || !layout_ok(&C->L)) return false;
  for (int c = 0; c < 3; ++c) {
    if (C->L.pool_pages[c] > 0 && (!C->pool[c] || !C->slot_pos[c])) return false;
    // page-head blocks are moved by bulk copies and 16-byte vector stores
    if (!aligned(C->pool[c], 16) || !aligned(C->slot_pos[c], 4)) return false;
  }
  if (!(C->block_table && C->num_blocks && C->free_slots && C->free_top && C->fifo &&
        C->fifo_head && C->fifo_tail && C->live_count && C->live_list && C->live_index &&
        C->num_live && C->page_bump && C->status))
    return false;
  // 64-bit words are updated with 64-bit atomics; the rest are int32 arrays
  return aligned(C->block_table, 8) && aligned(C->live_list, 8) && aligned(C->num_blocks, 4) &&
         aligned(C->free_slots, 4) && aligned(C->free_top, 4) && aligned(C->fifo, 4) &&
         aligned(C->fifo_head, 4) && aligned(C->fifo_tail, 4) && aligned(C->live_count, 4) &&
         aligned(C->live_index, 4) && aligned(C->num_live, 4) && aligned(C->page_bump, 4) &&
         aligned(C->status, 4);
}

CacheView view_of(const thinkv_cache* C) {
  CacheView v;
  v.L = C->L;
  for (int c = 0; c < 3; ++c) {
    v.pool[c] = C->pool[c];
    v.slot_pos[c] = C->slot_pos[c];
  }
  v.block_table = C->block_table;
  v.num_blocks = C->num_blocks;
  v.free_slots = C->free_slots;
  v.free_top = C->free_top;
  v.fifo = C->fifo;
  v.fifo_head = C->fifo_head;
  v.fifo_tail = C->fifo_tail;
  v.live_count = C->live_count;
  v.live_list = C->live_list;
  v.live_index = C->live_index;
  v.num_live = C->num_live;
  v.page_bump = C->page_bump;
  v.status = C->status;
  return v;
}

}  // namespace thinkv

namespace {

int num_sms_current() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (dev < 0 || dev >= 64) return 0;
  if (!cached[dev]) {
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    cached[dev] = sms;
  }
  return cached[dev];
}

}  // namespace

namespace thinkv {

int cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return THINKV_OK;
  if (getenv("THINKV_VERBOSE")) fprintf(stderr, "libthinkv: %s\n", cudaGetErrorString(e));
  return THINKV_ERR_CUDA;
}

}  // namespace thinkv

extern "C" {

int thinkv_layout_check(const thinkv_layout* L) {
  return layout_ok(L) ? THINKV_OK : THINKV_ERR_INVALID;
}

size_t thinkv_page_head_bytes(const thinkv_layout* L, int32_t cls) {
  if (!layout_ok(L) || cls < 0 || cls > 2) return 0;
  return (size_t)page_head_bytes(L->head_dim, L->group_size, L->bits[cls]);
}

size_t thinkv_buffer_bytes(const thinkv_layout* L, int32_t which) {
  if (!layout_ok(L)) return 0;
  const size_t ns = (size_t)L->max_seqs, nb = (size_t)L->max_blocks_per_seq;
  const size_t cap = nb * kPage;
  switch (which) {
    case THINKV_BUF_POOL_R:
    case THINKV_BUF_POOL_E:
    case THINKV_BUF_POOL_T: {
      const int c = which - THINKV_BUF_POOL_R;
      return (size_t)L->pool_pages[c] * L->num_kv_heads *
             (size_t)page_head_bytes(L->head_dim, L->group_size, L->bits[c]);
    }
    case THINKV_BUF_SLOT_POS_R:
    case THINKV_BUF_SLOT_POS_E:
    case THINKV_BUF_SLOT_POS_T:
      return (size_t)L->pool_pages[which - THINKV_BUF_SLOT_POS_R] * kPage * 4;
    case THINKV_BUF_BLOCK_TABLE: return ns * nb * 8;
    case THINKV_BUF_NUM_BLOCKS: return ns * 4;
    case THINKV_BUF_FREE_SLOTS: return ns * 3 * cap * 4;
    case THINKV_BUF_FREE_TOP: return ns * 3 * 4;
    case THINKV_BUF_FIFO: return ns * 3 * cap * 4;
    case THINKV_BUF_FIFO_HEAD: return ns * 3 * 4;
    case THINKV_BUF_FIFO_TAIL: return ns * 3 * 4;
    case THINKV_BUF_LIVE_COUNT: return ns * 4;
    case THINKV_BUF_LIVE_LIST: return ns * nb * 8;
    case THINKV_BUF_LIVE_INDEX: return ns * nb * 4;
    case THINKV_BUF_NUM_LIVE: return ns * 4;
    case THINKV_BUF_PAGE_BUMP: return 3 * 4;
    case THINKV_BUF_STATUS: return 4;
    default: return 0;
  }
}

int thinkv_cache_reset(const thinkv_cache* C, void* stream) {
  if (!cache_ok(C)) return THINKV_ERR_INVALID;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const thinkv_layout* L = &C->L;
  cudaError_t e = cudaSuccess;
  auto zero = [&](void* p, int which) {
    if (e == cudaSuccess && p) e = cudaMemsetAsync(p, 0, thinkv_buffer_bytes(L, which), s);
  };
  auto minus_one = [&](void* p, int which) {
    if (e == cudaSuccess && p) e = cudaMemsetAsync(p, 0xFF, thinkv_buffer_bytes(L, which), s);
  };
  zero(C->block_table, THINKV_BUF_BLOCK_TABLE);
  zero(C->num_blocks, THINKV_BUF_NUM_BLOCKS);
  zero(C->free_top, THINKV_BUF_FREE_TOP);
  zero(C->fifo_head, THINKV_BUF_FIFO_HEAD);
  zero(C->fifo_tail, THINKV_BUF_FIFO_TAIL);
  zero(C->live_count, THINKV_BUF_LIVE_COUNT);
  zero(C->num_live, THINKV_BUF_NUM_LIVE);
  zero(C->page_bump, THINKV_BUF_PAGE_BUMP);
  zero(C->status, THINKV_BUF_STATUS);
  minus_one(C->live_index, THINKV_BUF_LIVE_INDEX);
  for (int c = 0; c < 3; ++c)
    if (L->pool_pages[c] > 0) minus_one(C->slot_pos[c], THINKV_BUF_SLOT_POS_R + c);
  return cuda_status(e);
}

size_t thinkv_append_workspace_bytes(const thinkv_layout* L, int32_t n_tokens) {
  if (!layout_ok(L) || n_tokens < 0) return 0;
  return append_workspace_bytes(n_tokens);
}

int thinkv_append_quantize(const thinkv_cache* C, int32_t n, const int32_t* seq, const int32_t* pos,
                           const uint8_t* tag, const uint16_t* k, const uint16_t* v,
                           void* workspace, size_t workspace_bytes, void* stream) {
  if (!cache_ok(C) || n < 0) return THINKV_ERR_INVALID;
  if (n == 0) return THINKV_OK;
  if (!seq || !pos || !tag || !k || !v) return THINKV_ERR_INVALID;
  if (!aligned(seq, 4) || !aligned(pos, 4) || !aligned(k, 16) || !aligned(v, 16))
    return THINKV_ERR_INVALID;
  if (workspace && !aligned(workspace, 16)) return THINKV_ERR_INVALID;
  if (!workspace || workspace_bytes < append_workspace_bytes(n)) return THINKV_ERR_WORKSPACE;
  const int sms = num_sms_current();
  if (sms <= 0) return THINKV_ERR_CUDA;
  const AppendWorkspace ws = carve_append_workspace(workspace, n);
  return cuda_status(launch_append(view_of(C), n, seq, pos, tag, k, v, ws,
                                   static_cast<cudaStream_t>(stream), sms));
}

int thinkv_append_evict(const thinkv_cache* C, int32_t n, const int32_t* seq, const int32_t* pos,
                        const uint8_t* tag, const uint16_t* k, const uint16_t* v,
                        const int32_t* budget, const uint8_t* order, void* workspace,
                        size_t workspace_bytes, void* stream) {
  if (!cache_ok(C) || n < 0) return THINKV_ERR_INVALID;
  uint8_t o[3] = {THINKV_T, THINKV_E, THINKV_R};
  if (order) {
    for (int x = 0; x < 3; ++x) {
      if (order[x] > 2) return THINKV_ERR_INVALID;
      o[x] = order[x];
    }
    if (o[0] == o[1] || o[0] == o[2] || o[1] == o[2]) return THINKV_ERR_INVALID;
  }
  if (n == 0) return THINKV_OK;
  if (!seq || !pos || !tag || !k || !v || !budget) return THINKV_ERR_INVALID;
  if (!aligned(seq, 4) || !aligned(pos, 4) || !aligned(budget, 4) || !aligned(k, 16) ||
      !aligned(v, 16))
    return THINKV_ERR_INVALID;
  if (workspace && !aligned(workspace, 16)) return THINKV_ERR_INVALID;
  if (!workspace || workspace_bytes < append_workspace_bytes(n)) return THINKV_ERR_WORKSPACE;
  const int sms = num_sms_current();
  if (sms <= 0) return THINKV_ERR_CUDA;
  const AppendWorkspace ws = carve_append_workspace(workspace, n);
  return cuda_status(launch_append(view_of(C), n, seq, pos, tag, k, v, ws,
                                   static_cast<cudaStream_t>(stream), sms, budget, o));
}

int thinkv_evict(const thinkv_cache* C, int32_t n, const int32_t* seq, const int32_t* budget,
                 const uint8_t* order, void* stream) {
  if (!cache_ok(C) || n < 0) return THINKV_ERR_INVALID;
  uint8_t o[3] = {THINKV_T, THINKV_E, THINKV_R};
  if (order) {
    for (int x = 0; x < 3; ++x) {
      if (order[x] > 2) return THINKV_ERR_INVALID;
      o[x] = order[x];
    }
    if (o[0] == o[1] || o[0] == o[2] || o[1] == o[2]) return THINKV_ERR_INVALID;
  }
  if (n == 0) return THINKV_OK;
  if (!seq || !budget) return THINKV_ERR_INVALID;
  if (!aligned(seq, 4) || !aligned(budget, 4)) return THINKV_ERR_INVALID;
  return cuda_status(launch_evict(view_of(C), n, seq, budget, o, static_cast<cudaStream_t>(stream)));
}

size_t thinkv_tbe_buffer_bytes(const thinkv_layout* L, int32_t which) {
  if (!layout_ok(L)) return 0;
  const size_t ns = (size_t)L->max_seqs, cap = (size_t)L->max_blocks_per_seq * kPage;
  switch (which) {
    case THINKV_TBE_SEG: return ns * cap * 16;
    case THINKV_TBE_NSEG: return ns * 4;
    case THINKV_TBE_SETTLED: return ns * 4;
    default: return 0;
  }
}

static bool tbe_ok(const thinkv_tbe* T) {
  return T && T->seg && T->nseg && T->settled && aligned(T->seg, 16) && aligned(T->nseg, 4) &&
         aligned(T->settled, 4);
}

int thinkv_tbe_reset(const thinkv_layout* L, const thinkv_tbe* T, void* stream) {
  if (!layout_ok(L) || !tbe_ok(T)) return THINKV_ERR_INVALID;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(T->nseg, 0, thinkv_tbe_buffer_bytes(L, THINKV_TBE_NSEG), s);
  if (e == cudaSuccess)
    e = cudaMemsetAsync(T->settled, 0, thinkv_tbe_buffer_bytes(L, THINKV_TBE_SETTLED), s);
  return cuda_status(e);
}

size_t thinkv_tbe_workspace_bytes(int32_t n_tokens) {
  if (n_tokens < 0) return 0;
  return ((size_t)(n_tokens > 0 ? n_tokens : 1) * 4 + 255) / 256 * 256;
}

int thinkv_evict_tbe(const thinkv_cache* C, const thinkv_tbe* T, int32_t n, const int32_t* seq,
                     const int32_t* pos, const uint8_t* tag, int32_t t_min, const int32_t* schedule,
                     void* workspace, size_t workspace_bytes, void* stream) {
  if (!cache_ok(C) || !tbe_ok(T) || n < 0 || t_min < 0) return THINKV_ERR_INVALID;
  int32_t sch[3] = {64, 32, 16};
  if (schedule) {
    for (int k = 0; k < 3; ++k) {
      if (schedule[k] < 0) return THINKV_ERR_INVALID;
      sch[k] = schedule[k];
    }
  }
  if (n == 0) return THINKV_OK;
  if (!seq || !pos || !tag || !aligned(seq, 4) || !aligned(pos, 4)) return THINKV_ERR_INVALID;
  if (workspace && !aligned(workspace, 16)) return THINKV_ERR_INVALID;
  if (!workspace || workspace_bytes < thinkv_tbe_workspace_bytes(n)) return THINKV_ERR_WORKSPACE;
  return cuda_status(launch_tbe(view_of(C), reinterpret_cast<int4*>(T->seg), T->nseg, T->settled, n,
                                seq, pos, tag, t_min, sch, static_cast<int32_t*>(workspace),
                                static_cast<cudaStream_t>(stream)));
}

size_t thinkv_evict_slots_workspace_bytes(int32_t n_victims) {
  if (n_victims < 0) return 0;
  return ((size_t)(n_victims > 0 ? n_victims : 1) * 4 + 255) / 256 * 256;
}

int thinkv_evict_slots(const thinkv_cache* C, int32_t n, const int32_t* seq, const uint8_t* cls,
                       const int32_t* fifo_index, void* workspace, size_t workspace_bytes,
                       void* stream) {
  if (!cache_ok(C) || n < 0) return THINKV_ERR_INVALID;
  if (n == 0) return THINKV_OK;
  if (!seq || !cls || !fifo_index || !aligned(seq, 4) || !aligned(fifo_index, 4))
    return THINKV_ERR_INVALID;
  if (workspace && !aligned(workspace, 16)) return THINKV_ERR_INVALID;
  if (!workspace || workspace_bytes < thinkv_evict_slots_workspace_bytes(n)) return THINKV_ERR_WORKSPACE;
  return cuda_status(launch_evict_slots(view_of(C), n, seq, cls, fifo_index,
                                        static_cast<int32_t*>(workspace),
                                        static_cast<cudaStream_t>(stream)));
}

size_t thinkv_compact_workspace_bytes(int32_t n_seqs, int32_t max_tokens) {
  if (n_seqs < 0 || max_tokens < 0) return 0;
  return compact_workspace_bytes(n_seqs, max_tokens);
}

int thinkv_compact(const thinkv_cache* src, const thinkv_cache* dst, int32_t n, const int32_t* seq,
                   int32_t max_tokens, void* workspace, size_t workspace_bytes, void* stream) {
  if (!cache_ok(src) || !cache_ok(dst) || n < 0 || max_tokens < 0) return THINKV_ERR_INVALID;
  const thinkv_layout &A = src->L, &B = dst->L;
  if (A.num_q_heads != B.num_q_heads || A.num_kv_heads != B.num_kv_heads ||
      A.head_dim != B.head_dim || A.group_size != B.group_size || A.bits[0] != B.bits[0] ||
      A.bits[1] != B.bits[1] || A.bits[2] != B.bits[2] || A.fmt[0] != B.fmt[0] ||
      A.fmt[1] != B.fmt[1] || A.fmt[2] != B.fmt[2] || A.max_seqs != B.max_seqs ||
      A.max_blocks_per_seq != B.max_blocks_per_seq || n > A.max_seqs)
    return THINKV_ERR_INVALID;
  if (n == 0) return THINKV_OK;
  if (!seq || !aligned(seq, 4)) return THINKV_ERR_INVALID;
  if (workspace && !aligned(workspace, 16)) return THINKV_ERR_INVALID;
  if (!workspace || workspace_bytes < compact_workspace_bytes(n, max_tokens)) return THINKV_ERR_WORKSPACE;
  const int sms = num_sms_current();
  if (sms <= 0) return THINKV_ERR_CUDA;
  return cuda_status(launch_compact(view_of(src), view_of(dst), n, seq, max_tokens, workspace, sms,
                                    static_cast<cudaStream_t>(stream)));
}

size_t thinkv_decode_workspace_bytes(const thinkv_layout* L, int32_t n_seqs, int32_t topk) {
  if (!layout_ok(L) || n_seqs < 1 || n_seqs > 16384 || topk < 0 || topk > 64) return 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  DecodeLaunch dl;
  if (!plan_decode_launch(*L, n_seqs, topk, dev, &dl)) return 0;
  return decode_workspace_bytes(*L, n_seqs, topk, dl);
}

int thinkv_decode_attention(const thinkv_cache* C, int32_t n, const int32_t* seq,
                            const uint16_t* q, uint16_t* out, float* topk_mass, int32_t topk,
                            float softmax_scale, void* workspace, size_t workspace_bytes,
                            void* stream) {
  if (!cache_ok(C) || n < 1 || n > 16384) return THINKV_ERR_INVALID;
  if (!seq || !q || !out) return THINKV_ERR_INVALID;
  if (topk_mass && (topk < 1 || topk > 64)) return THINKV_ERR_INVALID;
  if (!decode_args_aligned(seq, q, out, topk_mass)) return THINKV_ERR_INVALID;
  if (workspace && !aligned(workspace, 16)) return THINKV_ERR_INVALID;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return THINKV_ERR_CUDA;
  DecodeLaunch dl;
  if (!plan_decode_launch(C->L, n, topk_mass ? topk : 0, dev, &dl)) return THINKV_ERR_INVALID;
  if (!workspace || workspace_bytes < decode_workspace_bytes(C->L, n, topk_mass ? topk : 0, dl))
    return THINKV_ERR_WORKSPACE;
  return cuda_status(launch_decode(view_of(C), n, seq, q, out, topk_mass, topk_mass ? topk : 0,
                                   softmax_scale, workspace, dl, static_cast<cudaStream_t>(stream)));
}

int thinkv_classify_thoughts(int32_t n, int32_t num_q_heads, const float* mass, float theta_t,
                             float theta_r, uint8_t* tags, void* stream) {
  if (n < 0 || num_q_heads < 1) return THINKV_ERR_INVALID;
  if (isnan(theta_t) || isnan(theta_r)) return THINKV_ERR_INVALID;
  if (n == 0) return THINKV_OK;
  if (!mass || !tags || !aligned(mass, 4)) return THINKV_ERR_INVALID;
  return cuda_status(launch_classify(n, num_q_heads, mass, theta_t, theta_r, tags,
                                     static_cast<cudaStream_t>(stream)));
}

int thinkv_get_status(const thinkv_cache* C, void* stream, int32_t* out) {
  if (!C || !C->status || !out) return THINKV_ERR_INVALID;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e == cudaSuccess) e = cudaMemcpy(out, C->status, sizeof(int32_t), cudaMemcpyDeviceToHost);
  return cuda_status(e);
}

int thinkv_clear_status(const thinkv_cache* C, void* stream) {
  if (!C || !C->status) return THINKV_ERR_INVALID;
  return cuda_status(cudaMemsetAsync(C->status, 0, sizeof(int32_t), static_cast<cudaStream_t>(stream)));
}

const char* thinkv_status_string(int32_t status) {
  switch (status) {
    case THINKV_OK: return "ok";
    case THINKV_ERR_INVALID: return "invalid argument or token data";
    case THINKV_ERR_OUT_OF_PAGES: return "page pool exhausted";
    case THINKV_ERR_OUT_OF_BLOCKS: return "block table full";
    case THINKV_ERR_CUDA: return "CUDA runtime error";
    case THINKV_ERR_TIMEOUT: return "bounded wait ran out";
    case THINKV_ERR_WORKSPACE: return "workspace missing or too small";
    default: return "unknown status";
  }
}

}  // extern "C"
