// thinkv_internal.h -- host/device structures shared by the libthinkv sources.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "thinkv.h"

namespace thinkv {

// The cache as kernels see it (passed by value).
struct CacheView {
  thinkv_layout L;
  uint8_t* pool[3];
  int32_t* slot_pos[3];
  uint64_t* block_table;
  int32_t* num_blocks;
  int32_t* free_slots;
  int32_t* free_top;
  int32_t* fifo;
  int32_t* fifo_head;
  int32_t* fifo_tail;
  int32_t* live_count;
  uint64_t* live_list;
  int32_t* live_index;
  int32_t* num_live;
  int32_t* page_bump;
  int32_t* status;
};

// One sequence run of an append call (slot-assignment scratch).
struct RunInfo {
  int32_t start, len, seq, pad;
  int32_t cnt[3];
  int32_t grants[3];
  int32_t page_base[3];
  int32_t pad2;
};

struct AppendWorkspace {
  uint32_t* arrive;   // arrival counter of the one-launch path (zero between calls)
  int32_t* ok;        // 1 once the slot assignment succeeded
  int32_t* tok_slot;  // [n] pool slot id (page*16 + slot) of every token
  RunInfo* runs;      // [n] sequence runs
};

size_t append_workspace_bytes(int32_t n);
AppendWorkspace carve_append_workspace(void* ws, int32_t n);
// budget (device, per token; the value at each run's first token counts) and
// order (host, 3 classes): the append is followed by an evict of each run's
// sequence to its budget, in one launch for calls of up to 512 tokens
cudaError_t launch_append(const CacheView& C, int32_t n, const int32_t* seq, const int32_t* pos,
                          const uint8_t* tag, const uint16_t* k, const uint16_t* v,
                          const AppendWorkspace& ws, cudaStream_t stream, int num_sms,
                          const int32_t* budget = nullptr, const uint8_t* order = nullptr);

cudaError_t launch_evict(const CacheView& C, int32_t n, const int32_t* seq, const int32_t* budget,
                         const uint8_t order[3], cudaStream_t stream);
// the evict of an append's runs: seq and budget are the append's token arrays
cudaError_t launch_evict_runs(const CacheView& C, int32_t n, const int32_t* seq, const int32_t* budget,
                              const uint8_t order[3], cudaStream_t stream);

// host-side checks shared by the entry points
inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }
bool cache_ok(const thinkv_cache* C);
CacheView view_of(const thinkv_cache* C);
// q rows and out rows are moved with bulk copies / 8-byte vector stores;
// seq and mass are plain 4-byte arrays
inline bool decode_args_aligned(const void* seq, const void* q, const void* out, const void* mass) {
  return aligned(seq, 4) && aligned(q, 16) && aligned(out, 16) && aligned(mass, 4);
}
// THINKV_OK, or THINKV_ERR_CUDA (printed to stderr when THINKV_VERBOSE is set)
int cuda_status(cudaError_t e);

// decode
struct DecodeLaunch {
  int grid;            // CTAs of the split kernel
  int warps_per_cta;
  int nstage;          // pipeline stages per warp
  int stage_bytes;     // bytes per stage
  size_t smem_bytes;   // dynamic shared memory of the split kernel
  int warp_smem;       // bytes of shared memory per warp
  int64_t pieces;      // piece records (warps + segments)
};
bool plan_decode_launch(const thinkv_layout& L, int32_t n_seqs, int32_t topk, int device,
                        DecodeLaunch* out);
size_t decode_workspace_bytes(const thinkv_layout& L, int32_t n_seqs, int32_t topk,
                              const DecodeLaunch& dl);
cudaError_t launch_decode(const CacheView& C, int32_t n, const int32_t* seq, const uint16_t* q,
                          uint16_t* out, float* mass, int32_t topk, float softmax_scale,
                          void* ws, const DecodeLaunch& dl, cudaStream_t stream);

// TBE (segment-level eviction on Transition thoughts)
cudaError_t launch_tbe(const CacheView& C, int4* seg, int32_t* nseg, int32_t* settled, int32_t n,
                       const int32_t* seq, const int32_t* pos, const uint8_t* tag, int32_t t_min,
                       const int32_t schedule[3], int32_t* run_start, cudaStream_t stream);

// explicit victims
cudaError_t launch_evict_slots(const CacheView& C, int32_t n, const int32_t* seq, const uint8_t* cls,
                               const int32_t* idx, int32_t* run_start, cudaStream_t stream);

// gather compaction (the step CT avoids; a baseline)
size_t compact_workspace_bytes(int32_t n, int32_t max_tokens);
cudaError_t launch_compact(const CacheView& S, const CacheView& Dc, int32_t n, const int32_t* seq,
                           int32_t max_tokens, void* workspace, int num_sms, cudaStream_t stream);

// thought classifier (mechanism only)
cudaError_t launch_classify(int32_t n, int32_t hq, const float* mass, float theta_t, float theta_r,
                            uint8_t* tags, cudaStream_t stream);

}  // namespace thinkv
