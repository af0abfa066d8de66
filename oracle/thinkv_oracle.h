/*
 * thinkv_oracle.h -- CPU oracle for the ThinKV decode hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * CPU-baseline / reference legs of bench.py may build, load or call this
 * code.  It shares nothing with the CUDA library (no headers, helpers or
 * tables) and is written to be checked by eye against the method it follows:
 *
 *   "ThinKV: Thought-Adaptive KV Cache Compression for Efficient Reasoning
 *   Models" -- arXiv abstract (paged decode attention in the PagedAttention
 *   style, slots freed by eviction reused, nothing compacted) and the explainer's
 *   "Resume Technique / Methodologie" sections: TBQ (precision assigned by
 *   thought type, R > E > T, group quantisation), TBE (eviction of tokens of
 *   less important thoughts) and "Implementation Systeme: Pensee Continue
 *   (CT)" (a block table extended with each slot's thought type, start
 *   index and eviction state; an evicted slot is refilled in place by a later
 *   token of the same type).
 *
 * Every place where the pages are silent is filled by one stated reading;
 * the list is kept with the design notes of this repository.
 *
 * Layout of the oracle's own state is deliberately "natural": one code per
 * (page, kv-head, K|V, slot, channel), one (scale, zero) pair per group.
 */
#ifndef THINKV_ORACLE_H
#define THINKV_ORACLE_H
#include <stdint.h>
#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { OR_OK = 0, OR_ERR_INVALID = 1, OR_ERR_OUT_OF_PAGES = 2, OR_ERR_OUT_OF_BLOCKS = 3 };
enum { OR_R = 0, OR_E = 1, OR_T = 2 };
#define OR_PAGE 16

/* code formats of a class (fmt[c]): integer asymmetric codes, or the float
 * formats the pages name for the class's bit width (8: FP8 E4M3, 4: FP4
 * E2M1, 2: ternary) */
enum { OR_FMT_INT = 0, OR_FMT_FLOAT = 1 };

typedef struct {
  int32_t num_q_heads, num_kv_heads, head_dim, page_size, group_size;
  int32_t bits[3];
  int32_t max_seqs, max_blocks_per_seq;
  int32_t pool_pages[3];
  int32_t fmt[3];
} or_layout;

typedef struct or_state or_state;

or_state* or_create(const or_layout* L);
void or_destroy(or_state* S);
const or_layout* or_get_layout(const or_state* S);

/* ---- the three operations ------------------------------------------- */
int or_append(or_state* S, int32_t n, const int32_t* seq, const int32_t* pos,
              const uint8_t* tag, const uint16_t* k_fp16, const uint16_t* v_fp16);
int or_evict(or_state* S, int32_t n, const int32_t* seq, const int32_t* budget,
             const uint8_t* order /* 3 classes, NULL = T,E,R */);
int or_decode(const or_state* S, int32_t n, const int32_t* seq,
              const uint16_t* q_fp16, double softmax_scale, int32_t topk,
              double* out /* [n][Hq][d] */, double* mass /* [n][Hq] or NULL */,
              int32_t threads);

/* TBE, segment-level eviction on Transition thoughts: called after or_append
 * with the same token arrays.  Each new T segment anneals the earlier
 * segments (R/E: keep schedule[level-1] tokens, level 1..3; T: keep the t_min
 * most recent earlier T tokens); evicted FIFO entries become tombstones (-1).
 * schedule: 3 retentions, NULL = {64, 32, 16}. */
int or_tbe(or_state* S, int32_t n, const int32_t* seq, const int32_t* pos, const uint8_t* tag,
           int32_t t_min, const int32_t* schedule);

/* Explicit victims: victim i is the token at FIFO counter idx[i] of the
 * class cls[i] FIFO of sequence seq[i] (head <= idx < tail), evicted in call
 * order (mask bit, start index -1, free-stack push, FIFO tombstone); a victim
 * whose entry is already a tombstone is skipped.  Invalid (nothing changes): a
 * sequence out of range, a class above 2, a counter outside the window, a
 * sequence whose victims are not contiguous in the call. */
int or_evict_slots(or_state* S, int32_t n, const int32_t* seq, const uint8_t* cls,
                   const int32_t* idx);

/* Gather compaction (what CT avoids): the live tokens of seq[0..n) move into
 * fresh hole-free pages of the empty cache dst (same geometry), class by
 * class, FIFO order within a class, codes copied. */
int or_compact(const or_state* src, or_state* dst, int32_t n, const int32_t* seq);

/* Thought decomposition from attention sparsity (mechanism only): per
 * sequence i, score = (sum over heads, in head order, of mass[i][h]) / hq in
 * fp32; tag T if score >= theta_t, else R if score >= theta_r, else E. */
void or_classify(int32_t n, int32_t hq, const float* mass, float theta_t, float theta_r,
                 uint8_t* tags);

/* ---- building blocks, exposed for the pin tests ---------------------- */
uint16_t or_f16_round_down(float x);
uint16_t or_f16_round_up(float x);
uint16_t or_f16_round_nearest(float x);
float or_f16_to_f32(uint16_t h);
void or_f16_round_array(const float* x, int64_t n, int32_t mode, uint16_t* out);
void or_quantize_group(const uint16_t* x, int32_t G, int32_t bits,
                       uint8_t* codes, uint16_t* scale, uint16_t* zero);
/* the same for any format (fmt OR_FMT_FLOAT: E4M3 / E2M1 / ternary) */
void or_quantize_group_fmt(const uint16_t* x, int32_t G, int32_t bits, int32_t fmt,
                           uint8_t* codes, uint16_t* scale, uint16_t* zero);
/* E4M3 / E2M1: value of a code, and fp32 -> code rounded to nearest, ties to
 * even, saturating to the largest finite value */
double or_e4m3_value(uint8_t code);
uint8_t or_e4m3_from_f32(float x);
double or_e2m1_value(uint8_t code);
uint8_t or_e2m1_from_f32(float x);

/* ---- state export (for comparisons) ----------------------------------- */
/* Natural layouts:
 *   codes[c]   : [pool_pages[c]][Hkv][2][16][d]      uint8 codes (bits<=8)
 *                or uint16 raw fp16 bits (bits==16)
 *   params[c]  : [pool_pages[c]][Hkv][2][16][d/G][2] uint16 fp16 (scale, zero)
 *   slot_pos[c]: [pool_pages[c]][16]                  int32, -1 when dead
 *   table      : [max_seqs][max_blocks]               uint64 page|class<<32|mask<<48
 *   num_blocks, live_count, num_live : [max_seqs]     int32
 *   free_slots, fifo : [max_seqs][3][max_blocks*16]   int32 (entry*16+slot)
 *   free_top, fifo_head, fifo_tail : [max_seqs][3]    int32
 *   live_list  : [max_seqs][max_blocks]               uint64 page|class<<32|entry<<40
 *                of the entries with a non-zero mask (first num_live[s] valid)
 *   live_index : [max_seqs][max_blocks]               int32 position in live_list or -1
 *   page_bump : [3]                                   int32
 *   seg        : [max_seqs][max_blocks*16][5]         int32 TBE segments:
 *                class, level, lo (FIFO counter of the first token), len, trim
 *   nseg       : [max_seqs]                           int32 segments per sequence
 * A FIFO entry of -1 is a tombstone (evicted by TBE, not yet popped).
 */
const void* or_codes(const or_state* S, int c);
const uint16_t* or_params(const or_state* S, int c);
const int32_t* or_slot_pos(const or_state* S, int c);
const uint64_t* or_table(const or_state* S);
const int32_t* or_num_blocks(const or_state* S);
const int32_t* or_free_slots(const or_state* S);
const int32_t* or_free_top(const or_state* S);
const int32_t* or_fifo(const or_state* S);
const int32_t* or_fifo_head(const or_state* S);
const int32_t* or_fifo_tail(const or_state* S);
const int32_t* or_live_count(const or_state* S);
const uint64_t* or_live_list(const or_state* S);
const int32_t* or_live_index(const or_state* S);
const int32_t* or_num_live(const or_state* S);
const int32_t* or_page_bump(const or_state* S);
const int32_t* or_seg(const or_state* S);
const int32_t* or_nseg(const or_state* S);

#ifdef __cplusplus
}
#endif
#endif
