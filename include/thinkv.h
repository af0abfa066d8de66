/*
 * thinkv.h -- C ABI of libthinkv.so: the ThinKV decode hot path on B200 (sm_100a).
 *
 * What the library computes follows "ThinKV: Thought-Adaptive KV Cache
 * Compression for Efficient Reasoning Models":
 *   - arXiv abstract: decode attention over paged KV memory in the style of
 *     PagedAttention, where slots freed by eviction go to later tokens and
 *     nothing is compacted;
 *   - explainer, Resume Technique > Methodologie > "Quantification Adaptative
 *     a la Pensee (TBQ)": token precision set by thought type, R > E > T, by
 *     group quantisation;
 *   - explainer, Methodologie > "Eviction Adaptative a la Pensee (TBE)":
 *     tokens of less important thoughts are evicted;
 *   - explainer, Methodologie > "Implementation Systeme: Pensee Continue (CT)":
 *     a block table extended with each slot's thought type, start index and
 *     eviction state; an evicted slot is refilled in place by a later token of
 *     the same type.
 * Where the pages leave a choice open (integer code format, rounding of the
 * fp16 scale/zero, free-list discipline, eviction order, the attention-mass
 * statistic) this header states the choice made.
 *
 * Conventions for every entry point
 *   - All array arguments are DEVICE pointers owned by the caller, except the
 *     ones documented as host arrays.  The library allocates nothing and keeps
 *     no global state, apart from the fixed scratch array of
 *     thinkv_decode_attention_noalloc.  fp16 values travel as uint16_t bit
 *     patterns.
 *   - Alignment: pool[c], k, v, q, out and every workspace start on a 16-byte
 *     boundary (they are moved by bulk copies and 16-byte vector accesses);
 *     block_table and live_list on an 8-byte boundary; every other array on
 *     the boundary of its element type.  A pointer that breaks this is
 *     rejected with THINKV_ERR_INVALID before anything is launched.
 *   - `stream` is a cudaStream_t passed as void*; every call is asynchronous
 *     on it.
 *   - Host-checkable errors (bad layout, null pointers, sizes) return a
 *     non-zero thinkv_status before anything is launched.
 *   - Device-detected errors (bad token/sequence data, exhausted page pool,
 *     full block table, a bounded wait that ran out) are written to the
 *     cache's sticky `status` word: the first error wins and later errors do
 *     not overwrite it.  While *status != 0, append and evict do nothing;
 *     decode still runs (it only reads state that every operation leaves
 *     consistent).  thinkv_get_status / thinkv_clear_status read and reset it.
 *   - Nothing traps or spins without a bound.
 *   - Small appends, small evicts and decode launch their kernels with
 *     programmatic stream serialisation: a kernel may start while the
 *     previous kernel on the stream is finishing.  Before waiting for that
 *     kernel it reads only the call's own input arrays (token ids,
 *     positions, tags, K/V rows, budgets, sequence ids); cache state is read
 *     after the wait.  The library's kernels never write a call's inputs.  A
 *     caller whose own kernel writes a call's inputs, directly before the
 *     call, must not release its dependents early
 *     (griddepcontrol.launch_dependents); a copy or an ordinary kernel
 *     completes before the call's kernels start.
 */
#ifndef THINKV_H
#define THINKV_H
#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define THINKV_API __attribute__((visibility("default")))
#else
#define THINKV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  THINKV_OK = 0,
  THINKV_ERR_INVALID = 1,        /* bad argument or token/sequence data           */
  THINKV_ERR_OUT_OF_PAGES = 2,   /* a class page pool is exhausted                */
  THINKV_ERR_OUT_OF_BLOCKS = 3,  /* a sequence's block table is full              */
  THINKV_ERR_CUDA = 4,           /* a CUDA runtime call failed                    */
  THINKV_ERR_TIMEOUT = 5,        /* a bounded wait inside a kernel ran out        */
  THINKV_ERR_WORKSPACE = 6       /* workspace missing or too small                */
} thinkv_status;

/* thought types (classes) */
enum { THINKV_R = 0, THINKV_E = 1, THINKV_T = 2 };
#define THINKV_PAGE_SIZE 16

/* Geometry of one cache (one attention layer); immutable after creation.
 *   num_q_heads % num_kv_heads == 0 and num_q_heads / num_kv_heads <= 8
 *   (query heads map contiguously onto kv-heads: q-head h uses kv-head
 *   h / (num_q_heads / num_kv_heads));
 *   head_dim in {64, 128}; group_size in {32, 64}, dividing head_dim;
 *   page_size == 16; bits[c] in {2, 4, 8, 16} for c = R, E, T;
 *   1 <= max_seqs <= 65536; 1 <= max_blocks_per_seq <= 2^21;
 *   num_kv_heads <= 256; 0 <= pool_pages[c] < 2^27;
 *   fmt[c] in {THINKV_FMT_INT, THINKV_FMT_FLOAT}, FLOAT only with bits 2, 4, 8. */
typedef struct {
  int32_t num_q_heads, num_kv_heads, head_dim, page_size, group_size;
  int32_t bits[3];
  int32_t max_seqs, max_blocks_per_seq;
  int32_t pool_pages[3];
  int32_t fmt[3];
} thinkv_layout;

/* Code formats of a class (fmt[c]).  THINKV_FMT_INT: integer asymmetric codes
 * (the quantiser below).  THINKV_FMT_FLOAT: the formats the explainer's TBQ
 * names, by bit width -- 8: FP8 E4M3, scale = fp16 rounded up of amax/448,
 * zero 0, code = E4M3 of fp32(x/scale); 4: FP4 E2M1 (NVFP4's element format;
 * the group of G channels with its fp16 scale stands in for NVFP4's
 * 16-element E4M3 micro-scales), scale = fp16 rounded up of amax/6, zero 0;
 * 2: ternary, scale = fp16 rounded up of amax, code = clamp(rint_even(fp32(x
 * / scale)), -1, 1) + 1, zero = -scale.  amax: the group's largest |x|.
 * E4M3/E2M1 rounding: to nearest, ties to even, saturating to 448 / 6.
 * Dequantised value: scale * value(code) (E4M3/E2M1), zero + code * scale
 * (ternary, as integer codes).  Same bytes and layout as the integer codes
 * of that width.  A zero-filled fmt is all integer. */
enum { THINKV_FMT_INT = 0, THINKV_FMT_FLOAT = 1 };

/* The cache: device buffers, all allocated and owned by the caller with the
 * sizes thinkv_buffer_bytes() reports, and initialised by thinkv_cache_reset().
 *
 *   pool[c]       uint8 [pool_pages[c]][num_kv_heads][page_head_bytes(c)]
 *                 One "page-head block" holds 16 token slots of one kv-head:
 *                 K codes, V codes, K params, V params (layout below).
 *   slot_pos[c]   int32 [pool_pages[c]][16]  position of the token in each slot
 *                 (the block table's "start index"), -1 when the slot is dead.
 *   block_table   uint64 [max_seqs][max_blocks_per_seq]
 *                 entry = page | class << 32 | live_mask << 48
 *                 (bit s of live_mask: slot s holds a live token; this is the
 *                 eviction mask, inverted).
 *   num_blocks    int32 [max_seqs]       entries in use per sequence
 *   free_slots    int32 [max_seqs][3][max_blocks_per_seq*16]  per (sequence,
 *                 class) LIFO stack of reusable slots; a slot id is
 *                 entry*16 + slot.   free_top int32 [max_seqs][3].
 *   fifo          int32 [max_seqs][3][max_blocks_per_seq*16]  per (sequence,
 *                 class) ring of live slot ids in arrival order;
 *                 fifo_head, fifo_tail int32 [max_seqs][3] monotone counters
 *                 (ring index = counter mod capacity).
 *   live_count    int32 [max_seqs]       live tokens per sequence
 *   live_list     uint64 [max_seqs][max_blocks_per_seq]  one descriptor
 *                 page | class << 32 | entry << 40 per table entry with a
 *                 non-zero live_mask (first num_live[s] valid); an entry joins
 *                 at the end when it gains its first live token and leaves by
 *                 swap-with-last when it loses its last one.
 *   live_index    int32 [max_seqs][max_blocks_per_seq]  position of an entry
 *                 in live_list, -1 if absent.    num_live int32 [max_seqs].
 *   page_bump     int32 [3]              pages handed out per class pool
 *   status        int32 [1]              sticky device status (thinkv_status)
 *
 * Page-head block of a class with b = bits[c] < 16 (d = head_dim, G =
 * group_size, ng = d/G), byte offsets:
 *   [0, 2db)          K codes      [2db, 4db)  V codes
 *   [4db, 4db+64ng)   K params     [4db+64ng, 4db+128ng)  V params
 * params: [group ng][slot 16][scale, zero] fp16.
 * Each code region (K, V) holds a portion of d*b/16 bytes for each of 32
 * lanes, l = 4*gid + tid (gid 0..7, tid 0..3).  The portions are interleaved
 * in chunks of u = min(16, d*b/16) bytes: byte o of lane l's portion is at
 * (o / u)*32*u + l*u + o % u of the region.  Within 32-bit words (or a 16-bit
 * piece) the codes of even channels sit in the low half and those of odd
 * channels in the high half, each half little-endian.
 *   K: lane l holds, for group gr = 0..ng-1 and r = 0..1, the codes of slot
 *      gid + 8r, channels gr*G + tid*G/4 .. +G/4 (a piece of G*b/32 bytes),
 *      pieces ordered (gr, r).
 *   V: lane l holds words ordered (P = 0..1, q = 0..d*b/128-1); word (P, q)
 *      has slot 2*tid + 8P in its low 16 bits and slot 2*tid + 8P + 1 in its
 *      high 16 bits; each half holds 16/b codes, element k of chunk q being
 *      channel 16*(e/2) + gid + 8*(e%2) with e = q*16/b + k.
 * For b == 16 the block is K raw fp16 [2db) then V raw fp16 [2db), in the same
 * lane orders and chunk interleave, with no params.
 *
 * Quantiser (reading of TBQ's group quantisation): per token, per kv-head,
 * per K|V, per group of G consecutive channels: zero = min rounded toward
 * -inf to fp16; scale = fp32((max - zero)/(2^b - 1)) rounded toward +inf to
 * fp16; code = clamp(rint_half_even(fp32(fp32(x - zero)/scale)), 0, 2^b-1),
 * all fp32 operations rounded to nearest; scale 0 gives code 0.  Dequantised
 * value: zero + code*scale.
 */
typedef struct {
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
} thinkv_cache;

/* buffer ids for thinkv_buffer_bytes */
enum {
  THINKV_BUF_POOL_R = 0, THINKV_BUF_POOL_E = 1, THINKV_BUF_POOL_T = 2,
  THINKV_BUF_SLOT_POS_R = 3, THINKV_BUF_SLOT_POS_E = 4, THINKV_BUF_SLOT_POS_T = 5,
  THINKV_BUF_BLOCK_TABLE = 6, THINKV_BUF_NUM_BLOCKS = 7,
  THINKV_BUF_FREE_SLOTS = 8, THINKV_BUF_FREE_TOP = 9,
  THINKV_BUF_FIFO = 10, THINKV_BUF_FIFO_HEAD = 11, THINKV_BUF_FIFO_TAIL = 12,
  THINKV_BUF_LIVE_COUNT = 13, THINKV_BUF_LIVE_LIST = 14, THINKV_BUF_LIVE_INDEX = 15,
  THINKV_BUF_NUM_LIVE = 16, THINKV_BUF_PAGE_BUMP = 17, THINKV_BUF_STATUS = 18,
  THINKV_NUM_BUFFERS = 19
};

/* THINKV_OK if the layout is supported, else THINKV_ERR_INVALID. */
THINKV_API int thinkv_layout_check(const thinkv_layout* L);

/* Bytes of one page-head block of class c (0 for a bad layout or class). */
THINKV_API size_t thinkv_page_head_bytes(const thinkv_layout* L, int32_t cls);

/* Bytes of buffer `which` (THINKV_BUF_*); 0 for a bad layout or id. */
THINKV_API size_t thinkv_buffer_bytes(const thinkv_layout* L, int32_t which);

/* Empties the cache on `stream`: no pages granted, no live tokens, all
 * slot_pos and live_index -1, status THINKV_OK.  Pool bytes are left as they
 * are (a slot's bytes are only read while the slot is live). */
THINKV_API int thinkv_cache_reset(const thinkv_cache* cache, void* stream);

/* Workspace bytes thinkv_append_quantize needs for n_tokens tokens. */
THINKV_API size_t thinkv_append_workspace_bytes(const thinkv_layout* L, int32_t n_tokens);

/* Quantize-on-append (TBQ + CT write path).
 * Appends n_tokens tokens: token i belongs to sequence seq[i] at position
 * pos[i] with thought type tag[i] (0 = R, 1 = E, 2 = T); k and v are fp16
 * [n_tokens][num_kv_heads][head_dim].  Tokens must come grouped by sequence
 * (one contiguous run per sequence per call, positions strictly ascending
 * within the run); positions should also grow across calls (they order the
 * tokens of a sequence).
 * Each token takes the top slot of its (sequence, class) free stack; when that
 * stack is empty the class pool grants the next page (page_bump[c]), a table
 * entry {page, class, mask 0} is appended, slots 15..1 are pushed (slot 1 on
 * top) and slot 0 is used.  The token's K and V are quantised at bits[class]
 * into the slot, its live bit and slot_pos are set, its slot id is pushed on
 * the (sequence, class) FIFO and live_count grows.  Grants follow call order.
 * The call is all-or-nothing: device-detected errors (seq out of range, tag >
 * 2, negative or non-ascending positions, a sequence in two runs ->
 * INVALID; pool exhausted -> OUT_OF_PAGES; table full -> OUT_OF_BLOCKS,
 * checked in that order) set *status and change nothing.
 * workspace: device, >= thinkv_append_workspace_bytes(L, n_tokens) bytes,
 * caller-owned scratch.  Its first 4 bytes are an arrival counter of the
 * one-launch path taken by calls of up to 512 tokens: zero-fill the workspace
 * once before its first use; every call leaves the counter zero (a call that
 * stops on a device-detected error stops before anything arrives).  The
 * rest needs no initialisation.  Calls that share a workspace must not
 * overlap on the GPU. */
THINKV_API int thinkv_append_quantize(const thinkv_cache* cache, int32_t n_tokens,
                           const int32_t* seq, const int32_t* pos, const uint8_t* tag,
                           const uint16_t* k, const uint16_t* v,
                           void* workspace, size_t workspace_bytes, void* stream);

/* Append + evict in one call: the tokens are appended exactly as by
 * thinkv_append_quantize, then each sequence of the call is evicted to its
 * budget exactly as by thinkv_evict with `order` (host array of the 3 classes
 * in victim order, NULL for T, E, R).  budget: device int32 [n_tokens], 4-byte
 * aligned; the value at the first token of each sequence's run is that
 * sequence's budget (>= 0), the others are not read.  The call is
 * all-or-nothing: bad token data or a negative budget -> *status = INVALID and
 * nothing changes (with the other errors of thinkv_append_quantize).  Calls of
 * up to 512 tokens take one launch: each sequence's evict runs in the CTA that
 * assigned its slots, right after the assignment, with no second kernel.
 * Larger calls take the append's two kernels and one evict kernel.
 * workspace: as for thinkv_append_quantize (same size, same counter rule). */
THINKV_API int thinkv_append_evict(const thinkv_cache* cache, int32_t n_tokens, const int32_t* seq,
                                   const int32_t* pos, const uint8_t* tag, const uint16_t* k,
                                   const uint16_t* v, const int32_t* budget, const uint8_t* order,
                                   void* workspace, size_t workspace_bytes, void* stream);

/* Evict to budget (TBE + CT free path).
 * For each i < n_seqs, sequence seq[i] (distinct, in range) keeps at most
 * budget[i] >= 0 live tokens: n = max(0, live_count - budget) victims are the
 * oldest live tokens of the first class in `order` whose FIFO is non-empty,
 * then the next class, and so on.  Each victim's live bit is cleared, its
 * slot_pos set to -1 and its slot pushed on its class's free stack, in victim
 * order; entries that lose their last live token leave live_list.  Pages stay
 * with their sequence (no compaction, no release).
 * order: HOST array of 3 distinct classes, or NULL for {T, E, R}.
 * Bad seq/budget data -> *status = INVALID and nothing changes. */
THINKV_API int thinkv_evict(const thinkv_cache* cache, int32_t n_seqs, const int32_t* seq,
                 const int32_t* budget, const uint8_t* order, void* stream);

/* TBE segment state of a cache (caller-owned device buffers, sizes from
 * thinkv_tbe_buffer_bytes, cleared by thinkv_tbe_reset together with a
 * thinkv_cache_reset of the cache):
 *   seg      int32 [max_seqs][max_blocks_per_seq*16][4]  one record per
 *            segment: class | level << 8, lo (FIFO counter of its first
 *            token), len (tokens), trim (how far from lo TBE has evicted)
 *   nseg     int32 [max_seqs]   segments recorded per sequence
 *   settled  int32 [max_seqs]   segments before it no T event can change
 *            any more (a speed-up: they are not visited again) */
typedef struct {
  int32_t* seg;
  int32_t* nseg;
  int32_t* settled;
} thinkv_tbe;

enum { THINKV_TBE_SEG = 0, THINKV_TBE_NSEG = 1, THINKV_TBE_SETTLED = 2, THINKV_TBE_NUM_BUFFERS = 3 };

/* Bytes of TBE buffer `which` (THINKV_TBE_*); 0 for a bad layout or id. */
THINKV_API size_t thinkv_tbe_buffer_bytes(const thinkv_layout* L, int32_t which);

/* Empties the TBE state (no segments) on `stream`. */
THINKV_API int thinkv_tbe_reset(const thinkv_layout* L, const thinkv_tbe* tbe, void* stream);

/* Workspace bytes thinkv_evict_tbe needs for n_tokens tokens. */
THINKV_API size_t thinkv_tbe_workspace_bytes(int32_t n_tokens);

/* TBE: segment-level eviction on Transition thoughts (explainer, Resume
 * Technique > Methodologie > "Eviction Adaptative a la Pensee (TBE)", and
 * "Astuce B": a small safety net of Transition tokens is always kept).
 * Call it right after thinkv_append_quantize with the same token arrays
 * (n_tokens, seq, pos, tag).  Readings: a segment is a maximal run of
 * consecutive tokens of a sequence with one tag; the first token of a new T
 * segment is a T event.  At each T event, in call order, every earlier R or
 * E segment takes the next step of `schedule` (its k-th event keeps at most
 * schedule[min(k,3)-1] of its tokens) and the earlier T segments keep only
 * the t_min most recent live T tokens among them.  A segment gives up its
 * oldest tokens first; victims go in segment order, then token order: each
 * one's live bit is cleared, its slot_pos set to -1, its slot pushed on its
 * class's free stack (CT: refilled in place later), and its FIFO entry
 * becomes a tombstone (-1) that thinkv_evict steps over.
 * schedule: HOST array of 3 retentions >= 0, or NULL for {64, 32, 16};
 * t_min >= 0.  Bad token data or a full segment table -> *status = INVALID
 * and nothing changes; while *status != 0 the call does nothing.
 * workspace: device, >= thinkv_tbe_workspace_bytes(n_tokens) bytes, no
 * initialisation needed.  One kernel. */
THINKV_API int thinkv_evict_tbe(const thinkv_cache* cache, const thinkv_tbe* tbe, int32_t n_tokens,
                                const int32_t* seq, const int32_t* pos, const uint8_t* tag,
                                int32_t t_min, const int32_t* schedule, void* workspace,
                                size_t workspace_bytes, void* stream);

/* Workspace bytes thinkv_evict_slots needs for n_victims victims. */
THINKV_API size_t thinkv_evict_slots_workspace_bytes(int32_t n_victims);

/* Explicit victims: the eviction step a policy drives when it chooses the
 * victims itself (explainer, Methodologie, "Eviction Adaptative a la Pensee
 * (TBE)": segment-level eviction chosen by a policy; "Implementation Systeme:
 * Pensee Continue (CT)": an evicted slot is marked in the block table and
 * refilled in place later).  Victim i is the token at FIFO counter
 * fifo_index[i] of the class cls[i] FIFO of sequence seq[i]; the counters of
 * a (sequence, class) FIFO run from fifo_head to fifo_tail - 1, in arrival
 * order.  Victims go in call order, each like a TBE victim: live bit cleared,
 * slot_pos -1, slot pushed onto its class's free stack, FIFO entry made a
 * tombstone (-1) that thinkv_evict steps over.  A victim whose entry is
 * already a tombstone (evicted before, or named earlier in the call) is
 * skipped.  A sequence out of range, a class above 2, a counter outside
 * [fifo_head, fifo_tail) or a sequence whose victims are not contiguous in the
 * call -> *status = INVALID and nothing changes; while *status != 0 the call
 * does nothing.  TBE counts a segment's live tokens as a suffix of it, so a
 * cache driven by thinkv_evict_tbe should not also take victims from inside
 * its segments.
 * seq, fifo_index: device int32 [n_victims] (4-byte aligned); cls: device
 * uint8 [n_victims].  workspace: device, >= thinkv_evict_slots_workspace_bytes
 * (n_victims) bytes, no initialisation needed.  One kernel. */
THINKV_API int thinkv_evict_slots(const thinkv_cache* cache, int32_t n_victims, const int32_t* seq,
                                  const uint8_t* cls, const int32_t* fifo_index, void* workspace,
                                  size_t workspace_bytes, void* stream);

/* Workspace bytes thinkv_compact needs for n_seqs sequences holding at most
 * max_tokens live tokens together. */
THINKV_API size_t thinkv_compact_workspace_bytes(int32_t n_seqs, int32_t max_tokens);

/* Gather compaction: the step Continuous Thinking avoids, as a baseline to
 * measure it by (explainer, Methodologie, "Implementation Systeme: Pensee
 * Continue (CT)": evicting scattered tokens leaves holes that a gather-based
 * compaction would close at a cost in time and HBM bandwidth; CT refills them
 * in place; Resultats: the TPOT gain comes mainly from not compacting).
 * The live tokens of seq[0..n_seqs) (distinct) in `src` move into fresh,
 * hole-free pages of `dst`, a cache of the same geometry (pool sizes may
 * differ) that holds nothing yet for those sequences: class by class (R, E,
 * T), FIFO order within a class, 16 to a page, codes and params copied (not
 * requantised), as if appended there in that order.  The last page of a class
 * keeps its unused slots on the free stack; src's tombstones and free slots
 * are not carried over; pages are granted in call order per class.  src is
 * only read.  Decode over dst gives the same attention as over src.
 * max_tokens: an upper bound of the live tokens of the listed sequences (a
 * larger count sets dst's *status = INVALID).  A non-empty dst sequence or a
 * repeated/out-of-range id -> INVALID, an exhausted dst pool -> OUT_OF_PAGES,
 * both in dst's status with nothing changed.  workspace: device, >=
 * thinkv_compact_workspace_bytes(n_seqs, max_tokens), no initialisation.
 * Four kernels: count (a warp per sequence and class), plan (one CTA), list
 * (a warp per sequence and class) and copy (a warp per page-head). */
THINKV_API int thinkv_compact(const thinkv_cache* src, const thinkv_cache* dst, int32_t n_seqs,
                              const int32_t* seq, int32_t max_tokens, void* workspace,
                              size_t workspace_bytes, void* stream);

/* Workspace bytes thinkv_decode_attention needs on the CURRENT device. */
THINKV_API size_t thinkv_decode_workspace_bytes(const thinkv_layout* L, int32_t n_seqs, int32_t topk);

/* Decode attention over the mixed-precision pages (the PagedAttention
 * extension).  For each i < n_seqs (seq[i] distinct or not) and each q-head
 * h: o = softmax(scale * q K^T) V over the live tokens of seq[i], with K, V
 * dequantised from their class's codes (raw for 16-bit classes); kv-head
 * h / (Hq/Hkv).  q: fp16 [n_seqs][num_q_heads][head_dim]; out: fp16, same
 * shape (a sequence with no live token gives zeros).  softmax_scale <= 0
 * means 1/sqrt(head_dim).
 * topk_mass: NULL, or fp32 [n_seqs][num_q_heads]: the share of the softmax
 * probability held by the topk (1..64) most probable live tokens (1 when the
 * sequence has <= topk live tokens, 0 when it has none).
 * workspace: device, >= thinkv_decode_workspace_bytes(L, n_seqs, topk) bytes,
 * caller-owned scratch for the split-K partial results; its contents need no
 * initialisation.  Calls that share a workspace must not overlap on the GPU.
 * Two kernels run per call: the split kernel over the live page-heads and the
 * combine of the segments it left in several pieces.
 * 1 <= n_seqs <= 16384. */
THINKV_API int thinkv_decode_attention(const thinkv_cache* cache, int32_t n_seqs, const int32_t* seq,
                            const uint16_t* q, uint16_t* out, float* topk_mass,
                            int32_t topk, float softmax_scale,
                            void* workspace, size_t workspace_bytes, void* stream);

/* Size of the library-owned scratch of thinkv_decode_attention_noalloc. */
#define THINKV_NOALLOC_SCRATCH_BYTES (16u << 20)

/* Decode attention without a caller-provided workspace -- the same operation,
 * arguments and results as thinkv_decode_attention, for callers that cannot
 * allocate device memory at the point where they decode: code running inside
 * a host framework that owns every device allocation and hands its plugins no
 * allocator, or latency-critical paths where cudaMalloc's implicit device-wide
 * synchronisation is not acceptable.  (The ThinKV pages have no counterpart;
 * this is an interface convenience of this library.)
 * The split-K scratch lives in one file-scope device array of
 * THINKV_NOALLOC_SCRATCH_BYTES bytes that every GPU loading the library holds
 * until the process exits.  A call whose scratch need (what
 * thinkv_decode_workspace_bytes reports for the same n_seqs and topk) exceeds
 * that size returns THINKV_ERR_WORKSPACE before launching anything.
 * The first call on a device looks up the array's device address (once per
 * device, with that device current); make that first call before any stream
 * capture.  The looked-up address belongs to the device's context of that
 * moment: after cudaDeviceReset() on a device, this entry point must not be
 * called on that device again in the same process.  Calls share the array: two calls that overlap on the GPU
 * (different streams, or different host threads) race and must not be
 * issued.  Nothing is allocated or freed. */
THINKV_API int thinkv_decode_attention_noalloc(const thinkv_cache* cache, int32_t n_seqs,
                                               const int32_t* seq, const uint16_t* q,
                                               uint16_t* out, float* topk_mass, int32_t topk,
                                               float softmax_scale, void* stream);

/* Thought tags from attention sparsity (mechanism only).
 * Explainer, Resume Technique > Methodologie > "Decomposition de la Pensee
 * via la Parcimonie de l'Attention": Transition thoughts have the sparsest
 * attention, then Reasoning, and Execution the least sparse.
 * For each i < n: score = (mass[i][0] + mass[i][1] + ... + mass[i][hq-1]) /
 * hq, the sum taken left to right and the division in fp32 (round to
 * nearest); tags[i] = THINKV_T if score >= theta_t, else THINKV_R if
 * score >= theta_r, else THINKV_E.
 * mass: device fp32 [n][num_q_heads], e.g. the topk_mass output of
 * thinkv_decode_attention; tags: device uint8 [n].  The thresholds are the
 * calibration (the pages leave it to a real model); NaN thresholds or
 * n < 0 or num_q_heads < 1 -> THINKV_ERR_INVALID.  One kernel, no state. */
THINKV_API int thinkv_classify_thoughts(int32_t n, int32_t num_q_heads, const float* mass,
                                        float theta_t, float theta_r, uint8_t* tags,
                                        void* stream);

/* Synchronises `stream`, then copies *status to *out (host). */
THINKV_API int thinkv_get_status(const thinkv_cache* cache, void* stream, int32_t* out);

/* Sets *status back to THINKV_OK (asynchronously on `stream`). */
THINKV_API int thinkv_clear_status(const thinkv_cache* cache, void* stream);

/* Static description of a status code. */
THINKV_API const char* thinkv_status_string(int32_t status);

#ifdef __cplusplus
}
#endif
#endif /* THINKV_H */
