/*
 * kvcomp_next.h — calls of libkvcomp.so beyond the compression path of
 * kvcomp.h, on the same conventions (caller-owned device buffers, no
 * allocation, asynchronous on `stream`, status codes of kvcomp.h):
 *
 *   kv_voxzip_pool -> VoxZip first stage: semantic-anchored pooling of the
 *        audio feature rows ("VoxZip: Semantic-Anchored Temporal KV Cache
 *        Compression for Long-Context Audio Inference", 方法概述和架构,
 *        first stage, steps one to three).
 *   kv_wnw_update, kv_wnw_recall -> WnW's anchor-chunk importance with top-3
 *        selection and release hysteresis, and the recall of the selected
 *        chunks of the tidal heads from their full copy in host memory
 *        ("WnW: Waxing-and-Waning KV Cache for Long-Form Speech LLMs",
 *        方法概述和架构 and 细节详述).
 *   kv_c3_build, kv_c3_step -> C3's key-space index (bisecting 2-means),
 *        shared-GQA cluster competition for a budget of B audio keys, exact
 *        attention over them and adaptive resolution (relevance EMA with
 *        split/merge exchanges) ("C3: Speech-Guided KV Retrieval for
 *        Long-Context SpeechLLM Inference").
 */
#ifndef KVCOMP_NEXT_H
#define KVCOMP_NEXT_H

#include "kvcomp.h"

#ifdef __cplusplus
extern "C" {
#endif

#define KV_VZ_MAX_L (1 << 24)        /* audio feature rows per sequence        */
#define KV_VZ_MAX_SEGMENTS 4096      /* ASR segments per sequence              */
#define KV_VZ_MAX_D 16384            /* feature width                          */

/* Device status bit of kv_voxzip_pool: a segment's text rows run past
 * n_text_rows; that segment's groups are written without the text add. */
#define KV_DEV_RANGE 0x8

/* One timestamped ASR segment (32 bytes, device memory). */
typedef struct {
  double tau_start;   /* segment start, seconds from the start of the audio */
  double tau_end;     /* segment end, seconds                                */
  float confidence;   /* ASR confidence of the segment                       */
  int32_t n_text;     /* L_t: text tokens of the segment                     */
  int32_t text_row;   /* row of E_T holding the segment's first text token   */
  int32_t reserved;   /* set to 0                                            */
} kv_asr_segment;

/*
 * kv_voxzip_pool — VoxZip's semantic-anchored audio compression of n_seq
 * sequences of audio feature rows (VoxZip, 方法概述和架构, first stage):
 *   1. a segment is kept when confidence > conf_min (compared in float32; 0.3
 *      on the page), n_text >= 1 and idx_end > idx_start, where
 *      idx = floor(L_a * tau / tau_total) in float64 (the product first), each
 *      clamped to [0, L_a]; it covers feature rows [idx_start, idx_end);
 *      kept segments are taken in order, and one that starts before the end
 *      of an earlier kept segment starts at that end;
 *   2. a kept segment of len rows forms n = min(n_text, len) groups, group j
 *      being rows [floor(j len / n), floor((j + 1) len / n)) from its start;
 *      its output row is the element-wise mean of the group (float32 sum in
 *      row order, one division) plus text row text_row + j of E_T (when E_T
 *      is not NULL), rounded once to dtype;
 *   3. rows no kept segment covers are copied unchanged; all output rows are
 *      in time order.
 * Arguments:
 *   L_a        host [n_seq]: feature rows per sequence, 1..KV_VZ_MAX_L; the
 *              sum below 2^31.
 *   tau_total  host [n_seq]: audio duration in seconds, finite and > 0.
 *   seg_off    host [n_seq + 1]: sequence s owns segs[seg_off[s] ..
 *              seg_off[s + 1]), at most KV_VZ_MAX_SEGMENTS; seg_off[0] = 0.
 *   d, dtype   feature width (d * element size a multiple of 16 bytes, at most
 *              KV_VZ_MAX_D) and KV_BF16 or KV_F32 for E_A, E_T and E_comp.
 *   segs       device [seg_off[n_seq]] segments.
 *   E_A        device [sum L_a][d]: sequence s at rows sum_{s'<s} L_a[s'].
 *   E_T        device [n_text_rows][d] text embeddings, or NULL (no add).
 *   E_comp     device [sum L_a][d] (output): sequence s writes out_len[s]
 *              rows from the same first row as its E_A; the rest untouched.
 *   src        device [sum L_a][3] int32 (output), per output row: first
 *              feature row (within the sequence), rows pooled into it, text
 *              row (-1 for a copied row).
 *   out_len    device [n_seq] int32 (output).
 *   status     device int32: KV_DEV_RANGE is OR-ed in (see above); may be
 *              NULL only when E_T is NULL.
 * E_A, E_T and E_comp must not overlap. Errors: KV_ERR_ARG, KV_ERR_CUDA.
 */
int kv_voxzip_pool(const int32_t* L_a, int32_t n_seq, const double* tau_total, const int32_t* seg_off, int32_t d,
                   int32_t dtype, float conf_min, const kv_asr_segment* segs, const void* E_A, const void* E_T,
                   int64_t n_text_rows, void* E_comp, int32_t* src, int32_t* out_len, int32_t* status,
                   void* stream);

/* ------------------------------------------------------------------------ */
/* WnW anchor chunks and tidal recall                                        */
/* ------------------------------------------------------------------------ */
#define KV_WNW_MAX_L (1 << 20)     /* audio rows per sequence             */
#define KV_WNW_MAX_TOP 8           /* chunks selected per step            */
#define KV_WNW_MAX_SLOTS 1024      /* block slots per (sequence, tidal row) */
#define KV_WNW_MAX_CHUNK 12288     /* rows per chunk                      */

/* The chunk rule, named as on the WnW page (4 s chunks every 2 s, top 3,
 * released after 3 unselected steps), in audio rows. */
typedef struct {
  int32_t chunk_len;     /* C: rows per chunk (4 s of audio), <= KV_WNW_MAX_CHUNK */
  int32_t chunk_stride;  /* S: rows between chunk starts (2 s); C % S == 0      */
  int32_t top_c;         /* chunks selected per step, 1..KV_WNW_MAX_TOP (3)     */
  int32_t release_after; /* unselected steps in a row before a chunk leaves (3) */
  int32_t n_slots;       /* block slots of the GPU copy per (sequence, tidal
                            row): top_c * release_after * C / S ..
                            KV_WNW_MAX_SLOTS                                    */
} kv_wnw_params;

/* Chunks of a sequence of L rows: M = 1 when L <= C, else ceil((L - C) / S) + 1;
 * chunk m covers rows [m S, min(m S + C, L)). Blocks: nb = ceil(L / S), block b
 * covers rows [b S, min((b + 1) S, L)); chunk m holds blocks m .. m + C/S - 1
 * (those below nb).
 * kv_wnw_chunk_count: sum of M over the batch; kv_wnw_state_ints: int32 words
 * of the state (per sequence: idle [M], block_slot [nb], slot_block [n_slots]).
 * Both return -1 on invalid arguments. */
int64_t kv_wnw_chunk_count(const int32_t* L, int32_t n_seq, const kv_wnw_params* p);
int64_t kv_wnw_state_ints(const int32_t* L, int32_t n_seq, const kv_wnw_params* p);

/* Sets every chunk and block of `state` (device, kv_wnw_state_ints words) to
 * "not resident" (-1). Errors: KV_ERR_ARG, KV_ERR_CUDA. */
int kv_wnw_init(const int32_t* L, int32_t n_seq, const kv_wnw_params* p, int32_t* state, void* stream);

/*
 * kv_wnw_update — one decode step of WnW's anchor-chunk rule for every
 * sequence (WnW, 方法概述和架构: anchor attention summed into time-chunk
 * importance, top 3 chunks recalled; 细节详述: 4 s / 2 s chunks, released
 * after 3 unselected steps in a row):
 *   score_m = sum over anchor rows a, then over rows j of chunk m, of s[a][j]
 *             (float64, in that order);
 *   the top_c largest scores are selected (ties to the lower chunk; every
 *   chunk when M <= top_c); a selected chunk's idle count becomes 0, a
 *   resident unselected chunk's count grows by 1 and the chunk leaves when it
 *   reaches release_after;
 *   a block is resident while a resident chunk holds it; blocks that stop
 *   being resident free their slots (release list), then the blocks that
 *   become resident take the lowest free slots in ascending block order
 *   (fetch list).
 * Arguments:
 *   L        host [n_seq]: audio rows per sequence, 1..KV_WNW_MAX_L.
 *   n_anchor anchor rows (KV heads) per sequence, 1..1024.
 *   s        device [sum_s n_anchor * L[s]] float32: sequence s's anchors one
 *            after another, each L[s] long: the step's attention mass of the
 *            anchor row on every audio row (e.g. summed over its query heads).
 *   state    device, kv_wnw_state_ints words (updated).
 *   score    device [kv_wnw_chunk_count] float64 (output): sequence after
 *            sequence.
 *   fetch    device [n_seq][top_c * C / S][2] int32 (output): (block, slot)
 *            pairs, first counts[s][0] valid.
 *   release  device [n_seq][top_c * C / S][2] int32 (output): (block, old
 *            slot) pairs, first counts[s][1] valid.
 *   counts   device [n_seq][2] int32 (output).
 * Errors: KV_ERR_ARG, KV_ERR_CUDA.
 */
int kv_wnw_update(const int32_t* L, int32_t n_seq, const kv_wnw_params* p, int32_t n_anchor, const float* s,
                  int32_t* state, double* score, int32_t* fetch, int32_t* release, int32_t* counts, void* stream);

/*
 * kv_wnw_recall — copies the blocks of the fetch lists of kv_wnw_update from
 * the tidal rows' full K/V copies in host memory into their GPU copies (WnW,
 * 方法概述和架构: tidal heads keep the full KV on the CPU and hold only the
 * recalled chunks on the GPU). One kernel reads the host memory directly
 * (pinned, mapped) with 16-byte loads; the caller picks the stream, so the
 * copy can run beside the decode step.
 *   L, n_seq, p        as kv_wnw_update.
 *   n_tidal            tidal rows per sequence, >= 1.
 *   d, dtype           row width (d * element size a multiple of 16 bytes) and
 *                      KV_BF16 or KV_F32.
 *   fetch, counts      device, from kv_wnw_update.
 *   K_host, V_host     pinned host memory (cudaHostAlloc or registered),
 *                      [sum_s n_tidal * L[s]][d]: sequence s's tidal rows one
 *                      after another, each L[s] long.
 *   K_gpu, V_gpu       device [n_seq * n_tidal * n_slots * S][d]: slot k of
 *                      tidal row r of sequence s starts at row
 *                      ((s * n_tidal + r) * n_slots + k) * S; a short last
 *                      block leaves the rest of its slot untouched.
 * Errors: KV_ERR_ARG (also when K_host or V_host is not pinned host memory),
 * KV_ERR_CUDA.
 */
int kv_wnw_recall(const int32_t* L, int32_t n_seq, const kv_wnw_params* p, int32_t n_tidal, int32_t d, int32_t dtype,
                  const int32_t* fetch, const int32_t* counts, const void* K_host, const void* V_host, void* K_gpu,
                  void* V_gpu, void* stream);

/* ------------------------------------------------------------------------ */
/* C3 key-space retrieval                                                    */
/* ------------------------------------------------------------------------ */
#define KV_C3_MAX_BUDGET 8192 /* B, at most */

/* The method's settings, named as on the C3 page (defaults in brackets). */
typedef struct {
  int32_t leaf_max;    /* a node with more keys is split (4)                   */
  int32_t iters;       /* 2-means iterations per split (8), 1..64              */
  int32_t granularity; /* mean node size of the initial frontier (16), >= 4    */
  int32_t budget;      /* B: audio keys retrieved per row and step, 1..KV_C3_MAX_BUDGET */
  double lambda;       /* weight of the history in the relevance EMA (0.5)     */
  int32_t exchanges;   /* R: split/merge exchanges per step (2), 0..64         */
  int32_t reserved;    /* set to 0                                             */
  uint64_t seed;       /* seed of the 2-means initialisation (0)               */
} kv_c3_params;

/* Where each array of a C3 index lives, as byte offsets into the index buffer.
 * Per-key arrays hold row i at key offset koff_i (kvcomp.h's convention), per-
 * node arrays at 2 * koff_i (a row has at most 2 L nodes), cent at
 * 2 * koff_i * d; hdr is [rows][4] int32: node count, frontier size A,
 * retrieved keys, 0. */
typedef struct {
  uint64_t perm;  /* int32 per key: positions in index order                   */
  uint64_t lo;    /* int32 per node: first index of the node's members         */
  uint64_t cnt;   /* int32 per node: members                                   */
  uint64_t left;  /* int32 per node: left child (right = left + 1), or -1      */
  uint64_t depth; /* int32 per node                                            */
  uint64_t e;     /* float64 per node: relevance EMA                           */
  uint64_t cent;  /* float64 per node x d: centroid                            */
  uint64_t front; /* int32 per node: the frontier's node ids, ascending        */
  uint64_t sigma; /* float64 per node: the last step's score of frontier entry */
  uint64_t sel;   /* int32 per key: the last step's retrieved positions        */
  uint64_t hdr;   /* int32 [rows][4]                                           */
  uint64_t bytes; /* size of the whole index                                   */
} kv_c3_layout;

/* Layout of the index of a batch; KV_ERR_ARG on invalid arguments. */
int kv_c3_index_layout(const kv_shape* shape, const int32_t* L, int32_t n_seq, const kv_c3_params* p,
                       kv_c3_layout* out);

/*
 * kv_c3_build — prefill: the key-space index of every row (C3, index built
 * per layer and KV head by recursive bisecting k-means, 8 iterations, seed 0;
 * initial frontier at mean granularity 16):
 *   a node with more than leaf_max keys is split by 2-means (squared
 *   Euclidean distance in float64, ties to the left child) started from two
 *   distinct members picked by SplitMix64 (outputs 2n and 2n + 1 of the
 *   generator seeded with `seed`, n = the node's id in its row); an empty side
 *   keeps its centroid; a split that leaves a side empty halves the members;
 *   node ids are breadth-first; a node's members, in index order, are its left
 *   child's then its right child's (a leaf's in ascending position); its
 *   centroid is their mean (float64, summed in index order); the frontier is
 *   every node at depth round(log2(L / granularity)) plus the leaves above it;
 *   every EMA starts at 0.
 *   K      device [sum L][d] in shape->dtype (d = head_dim).
 *   index  device, kv_c3_index_layout().bytes, 8-byte aligned.
 * Runs one launch per tree level and synchronises `stream` after each (the
 * level count depends on the data). Errors: KV_ERR_ARG, KV_ERR_UNSUPPORTED_L,
 * KV_ERR_CUDA.
 */
int kv_c3_build(const kv_shape* shape, const int32_t* L, int32_t n_seq, const kv_c3_params* p, const void* K,
                void* index, void* stream);

/*
 * kv_c3_step — one decode step of every row (C3: shared-GQA competition over
 * the frontier, exact attention over the retrieved keys, adaptive resolution):
 *   sigma_n = max over the g query heads of cos(q_g, c_n) (float64);
 *   frontier clusters in descending sigma (ties: lower node id) give their
 *   members in index order until B keys are taken;
 *   out_g = softmax(q_g K_sel^T / sqrt(d)) V_sel over the retrieved keys
 *   (float32 accumulation);
 *   e_n = lambda e_n + (1 - lambda) sigma_n on the frontier, then R exchanges:
 *   the frontier node with children and the largest e (ties: lower id) is
 *   replaced by its children (which take its e), and the sibling pair on the
 *   frontier with the smallest max(e) (ties: lower parent id), not holding
 *   that node, by its parent (which takes that max); nodes made in the same
 *   step are not candidates; an exchange lacking either is skipped.
 *   A row with L <= B attends over all its keys and keeps its state.
 *   K, V   device [sum L][d]; q device [rows][g][d]; out device [rows][g][d],
 *          all in shape->dtype. index from kv_c3_build with the same shape,
 *          lengths and parameters (updated; not checked against them).
 * Errors: KV_ERR_ARG, KV_ERR_UNSUPPORTED_L, KV_ERR_CUDA.
 */
int kv_c3_step(const kv_shape* shape, const int32_t* L, int32_t n_seq, const kv_c3_params* p, const void* K,
               const void* V, const void* q, void* index, void* out, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* KVCOMP_NEXT_H */
