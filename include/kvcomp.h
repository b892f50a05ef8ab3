/*
 * kvcomp.h — C ABI of the B200 (sm_100a) library for attention-score-driven
 * KV-cache selection and compaction over long audio contexts.
 *
 * The path, per (sequence, layer, KV head) "row", is:
 *   kv_score  -> raw window importance scores s        (AudioKV blog §1.2)
 *   kv_sss    -> Spectral Score Smoothing s_hat, k*    (AudioKV blog §2.2)
 *   kv_allocate -> head-aware per-row budgets b        (AudioKV blog §3.1, §5.1)
 *   kv_select_gather -> kept indices + compacted K/V   (AudioKV blog §3.1)
 *   variants: kv_allocate_global (budgets pooled over a sequence's layers,
 *   AudioKV blog §2.1), kv_select_gather_segmented (WnW segment-wise subset)
 *   kv_decode_attn_update -> one decode step with the temporally decayed
 *        score update and sink/recent/top-N eviction   (VoxZip, second stage)
 *
 * Conventions shared by every call
 * --------------------------------
 * - Rows. A batch holds n_seq sequences (1 <= n_seq <= KV_MAX_SEQ); sequence
 *   s has L[s] audio keys (host array). Each sequence has n_layers *
 *   n_kv_heads rows; row index = (s * n_layers + layer) * n_kv_heads + head.
 * - Per-key tensors are concatenated over rows: row i occupies keys
 *   [koff_i, koff_i + L_i) where koff_i = sum of L over the rows before it.
 *   K and V are [sum L][d]; s and s_hat are [sum L] float32.
 * - Device pointers are caller-owned; the library allocates nothing, never
 *   synchronises the stream and keeps no state between calls. Every call is
 *   asynchronous on `stream` (a cudaStream_t; NULL = legacy default stream).
 * - Q/K/V/compacted caches/outputs use shape->dtype (KV_BF16 or KV_F32);
 *   scores, A and all accumulation are float32.
 * - Pointers must be 16-byte aligned; rows are dense and contiguous.
 * - Argument errors return a status synchronously and launch nothing.
 *   Errors found on the device (a bounded wait that ran out, a budget with
 *   no evictable middle) are OR-ed into a caller-owned device status word
 *   (see kv_read_device_status); a kernel that hits one returns early.
 * - Supported: head_dim 64 or 128; R = group * w <= 256; L[s] even, >= w,
 *   <= 32768, with no prime factor above 7 in L[s] / 2.
 */
#ifndef KVCOMP_H
#define KVCOMP_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define KV_MAX_SEQ 64
#define KV_MAX_L 32768

/* Status codes (return values and device status bits). */
enum {
  KV_OK = 0,
  KV_ERR_ARG = 1,           /* null/misaligned pointer, bad shape or size   */
  KV_ERR_UNSUPPORTED_L = 2, /* odd L, L > KV_MAX_L, prime factor > 7, L < w */
  KV_ERR_BUDGET = 3,        /* budget below H*w, or no evictable middle     */
  KV_ERR_WORKSPACE = 4,     /* workspace missing or smaller than required   */
  KV_ERR_CUDA = 5,          /* a CUDA runtime call failed                   */
  KV_ERR_TIMEOUT = 6        /* a bounded device wait ran out                */
};

/* Device status bits (OR-ed into the status word). */
#define KV_DEV_TIMEOUT 0x1
#define KV_DEV_BUDGET 0x2
#define KV_DEV_CAPACITY 0x4 /* a row holds more slots than the launch was sized for */
#define KV_DEV_BOUNDS 0x10  /* debug builds: a checked index fell outside its buffer */

enum { KV_F32 = 0, KV_BF16 = 1 };

/* Model-side shape of one batch. */
typedef struct {
  int32_t n_layers;   /* layers per sequence                         */
  int32_t n_kv_heads; /* H: KV heads per layer                        */
  int32_t group;      /* g: query heads per KV head (GQA group size)  */
  int32_t head_dim;   /* d: 64 or 128                                 */
  int32_t w;          /* observation window = local window (AudioKV §5.1 min_window) */
  int32_t dtype;      /* KV_BF16 or KV_F32                            */
} kv_shape;

/* The method's parameters, named as on the pages. */
typedef struct {
  int32_t budget_pct; /* kept fraction of the audio keys, percent, 1..100 (AudioKV §5.1 compression_ratio) */
  float alpha;        /* SSS blend weight (AudioKV §2.2, §5.1 sss.alpha)       */
  float rho;          /* SSS energy cutoff ratio (AudioKV §2.2, §5.1 cutoff_ratio) */
  float r;            /* base share of the allocation (AudioKV §3.1, base_ratio) */
  float gamma;        /* decay of the cumulative attention A (VoxZip, gamma = 0.95) */
  int32_t sinks_T;    /* attention sinks always kept (VoxZip, T = 4)           */
  int32_t recent_pct; /* recent window as percent of the budget (VoxZip, 20%)  */
} kv_params;

/* Decode-time compacted cache (all device pointers, caller-owned).
 * Row i owns slots [slot_off[i], slot_off[i+1]) = b_i + 1 slots: b_i kept
 * entries plus one slot for the appended token. The cache is slot-stable:
 * an appended token takes the slot freed by the previous eviction, and the
 * logical order of entries is their position `pos`, not their slot. */
typedef struct {
  void* Kc;                /* [total_slots][d] dtype                      */
  void* Vc;                /* [total_slots][d] dtype                      */
  float* A;                /* [total_slots] decayed cumulative attention  */
  int32_t* pos;            /* [total_slots] audio/token position of the entry */
  const int64_t* slot_off; /* [rows + 1] from kv_allocate                 */
  const int32_t* b;        /* [rows] budgets from kv_allocate             */
  int32_t* meta;           /* [rows][8]: count, next free slot, steps done, last evicted slot,
                              prefill count, 3 reserved */
  int32_t* status;         /* device status word (KV_DEV_* bits)          */
  int64_t total_slots;     /* host: rows of Kc/Vc (slot_off[rows]); 0 = kv_total_slots() */
  void* scratch;           /* device, kv_decode_scratch_bytes() bytes (bf16 caches with group <= 8;
                              may be NULL otherwise): work items, per-slot logits, softmax
                              partials and their per-row lists, per-row step counters. Owned by
                              the caller, written by kv_decode_init, carried between steps.   */
  size_t scratch_bytes;
} kv_cache;

/* Number of rows of a batch. Returns -1 on a bad shape. */
int64_t kv_rows(const kv_shape* shape, int32_t n_seq);

/* Checks L[] against the supported lengths; KV_OK or KV_ERR_UNSUPPORTED_L. */
int kv_check_lengths(const kv_shape* shape, const int32_t* L, int32_t n_seq);

/* Bytes of device workspace kv_score needs for this batch (host query). */
size_t kv_workspace_bytes(const kv_shape* shape, const int32_t* L, int32_t n_seq);

/* Total compacted-cache slots sum_i (b_i + 1) for this batch (host query;
 * sum_h b_{l,h} = floor(budget_pct * L * H / 100) per layer), or -1. */
int64_t kv_total_slots(const kv_shape* shape, const int32_t* L, int32_t n_seq, const kv_params* params);

/* Bytes of decode scratch (kv_cache.scratch) for this batch and cache size
 * (0 when the cache is fp32 or group > 8: that path needs none). */
size_t kv_decode_scratch_bytes(const kv_shape* shape, const int32_t* L, int32_t n_seq, const kv_params* params,
                               int64_t total_slots);

/*
 * kv_score — observation-window importance scores (AudioKV blog §1.2: the raw
 * importance scores that SSS later smooths; SnapKV-style window scoring).
 *   s_j = sum_{r < R} softmax_j( q_r . K_j / sqrt(d) ),  R = group * w,
 * the softmax taken over all L keys of the row (no causal mask), summed over
 * the w window queries of each of the g query heads of the KV head.
 *   qwin : device, [rows][R][d] dtype; query head major (q of head g', window
 *          step i at R-index g' * w + i).
 *   K    : device, [sum L][d] dtype.
 *   s    : device, [sum L] float32 (output).
 *   ws   : device workspace of at least kv_workspace_bytes() bytes; its first
 *          4 bytes are the device status word of this call (cleared here).
 * Errors: KV_ERR_ARG, KV_ERR_UNSUPPORTED_L, KV_ERR_WORKSPACE, KV_ERR_CUDA.
 */
int kv_score(const kv_shape* shape, const int32_t* L, int32_t n_seq, const void* qwin, const void* K, float* s,
             void* ws, size_t ws_bytes, void* stream);

/*
 * kv_sss — Spectral Score Smoothing of every row (AudioKV blog §2.2):
 *   F = RFFT(s) (bins 0..L/2);  E(k) = sum_{i<=k} |F_i|^2;
 *   k* = min{ k : E(k) >= rho * E(L/2) };
 *   s_hat = (1 - alpha) s + alpha * IRFFT(F * 1[i <= k*], n = L).
 *   s, s_hat : device, [sum L] float32 (may not alias).
 *   kstar    : device, [rows] int32 (output).
 * Errors: KV_ERR_ARG, KV_ERR_UNSUPPORTED_L, KV_ERR_CUDA.
 */
int kv_sss(const kv_shape* shape, const int32_t* L, int32_t n_seq, const float* s, float* s_hat, int32_t* kstar,
           float alpha, float rho, void* stream);

/*
 * kv_allocate — head-aware budget allocation per (sequence, layer)
 * (AudioKV blog §3.1, defaults §5.1):
 *   B = floor(budget_pct * L * H / 100);  B_rem = B - H * w;
 *   x_h = w + r * B_rem / H + (1 - r) * B_rem * S_h / sum_h S_h;
 *   b_h = floor(x_h), the remainder +1 to the largest fractional parts (ties
 *   to the lower head), heads above L capped at L with the rest re-allocated
 *   over the other heads; sum_h S_h = 0 splits evenly.
 *   Computed in float64, every operation rounded to nearest on its own (no
 *   fused multiply-add), in this order, so the result is reproducible bit for
 *   bit: sumS = ((S_0 + S_1) + S_2) + ... in head order; t1 = r * B_rem;
 *   t1 = t1 / H; t2 = (1 - r) * B_rem; t2 = t2 * S_h; t2 = t2 / sumS;
 *   x_h = (w + t1) + t2 (r and S_h widened exactly from float32).
 *   S        : device, [n_layers][H] float32 per-head audio relevance.
 *   b        : device, [rows] int32 (output).
 *   slot_off : device, [rows + 1] int64 (output): prefix of b_i + 1.
 * Errors: KV_ERR_ARG, KV_ERR_BUDGET (B < H * w for some sequence), KV_ERR_CUDA.
 */
int kv_allocate(const kv_shape* shape, const int32_t* L, int32_t n_seq, const kv_params* params, const float* S,
                int32_t* b, int64_t* slot_off, void* stream);

/*
 * kv_allocate_global — the same allocation over every (layer, head) of a
 * sequence at once (AudioKV blog §2.1: the audio-critical heads concentrate
 * in some layers, so a budget shared across layers can follow them): the
 * n_layers * H heads share B = n_layers * floor(budget_pct * L * H / 100),
 * with the formula, rounding, remainder (ties to the lower (layer, head)) and
 * capping of kv_allocate over n_layers * H heads. The total per sequence, and
 * so kv_total_slots, is kv_allocate's.
 *   Arguments and outputs as kv_allocate; n_layers * n_kv_heads <= 1024.
 * Errors: KV_ERR_ARG, KV_ERR_BUDGET, KV_ERR_CUDA.
 */
int kv_allocate_global(const kv_shape* shape, const int32_t* L, int32_t n_seq, const kv_params* params,
                       const float* S, int32_t* b, int64_t* slot_off, void* stream);

/*
 * kv_select_gather — per-row selection and compaction (AudioKV blog §3.1
 * keeps the local window; the C3 page's bypass keeps all when b >= L):
 *   keep the last w positions and the top-(b - w) positions of s_hat over
 *   [0, L - w) (ties to the lower index), in ascending order; then
 *   Kc[slot_off_i + t] = K[koff_i + idx_t], same for V.
 *   s_hat : device, [sum L] float32;  K, V : [sum L][d] dtype, device memory or
 *           pinned (page-locked) host memory: only the b kept rows of each row are
 *           read, so K or V left on the host cross the host link b rows at a time.
 *   b, slot_off : device, from kv_allocate.
 *   idx   : device, [total_slots] int32 (output; row i writes b_i entries at
 *           slot_off[i]; the spare slot is left untouched). idx doubles as
 *           the initial `pos` array of the decode cache.
 *   Kc, Vc : device, [total_slots][d] dtype (output, same slots).
 *   A row with b < w (never produced by kv_allocate) is left unwritten.
 * Errors: KV_ERR_ARG (also for K or V in pageable host memory), KV_ERR_UNSUPPORTED_L, KV_ERR_CUDA.
 */
int kv_select_gather(const kv_shape* shape, const int32_t* L, int32_t n_seq, const float* s_hat, const void* K,
                     const void* V, const int32_t* b, const int64_t* slot_off, int32_t* idx, void* Kc, void* Vc,
                     void* stream);

/*
 * kv_select_gather_segmented — kv_select_gather with WnW's segment-wise
 * static subset (WnW digest: fixed heads keep positions chosen per segment,
 * not by one top-k over the whole recording, so no stretch is left without
 * cache): the candidates [0, L - w) are cut into n_segments segments
 * [floor(i (L - w) / n), floor((i + 1) (L - w) / n)); segment i keeps
 * q_i = floor(k len_i / (L - w)) of the k = b - w kept candidates, plus one
 * for the (k - sum q) segments with the largest remainders k len_i mod (L - w)
 * (ties to the lower segment), choosing its top-q_i by s_hat (ties to the
 * lower index). The window, the b >= L bypass, the outputs, the gather and
 * where K and V may live are those of kv_select_gather. 1 <= n_segments <=
 * 4096; n_segments = 1 is kv_select_gather.
 * Errors: KV_ERR_ARG, KV_ERR_CUDA.
 */
int kv_select_gather_segmented(const kv_shape* shape, const int32_t* L, int32_t n_seq, const float* s_hat,
                               const void* K, const void* V, const int32_t* b, const int64_t* slot_off,
                               int32_t n_segments, int32_t* idx, void* Kc, void* Vc, void* stream);

/*
 * kv_decode_init — prepares the decode state after kv_select_gather:
 *   A = 0 on every slot (VoxZip defines A by the decode recursion only),
 *   meta_i = {count = b_i, next free slot = b_i, steps = 0, last evicted = -1,
 *   prefill count = b_i}, builds the decode work items (rows cut into
 *   128-slot chunks) and clears the step counters in the scratch, and checks that every row has an evictable middle
 *   once a token is appended (b_i >= T + M_i) where
 *   M_i = floor(recent_pct * b_i / 100); rows without one set KV_DEV_BUDGET.
 * Errors: KV_ERR_ARG, KV_ERR_WORKSPACE (scratch missing or too small), KV_ERR_CUDA.
 */
int kv_decode_init(const kv_shape* shape, const int32_t* L, int32_t n_seq, const kv_params* params,
                   kv_cache* cache, void* stream);

/*
 * kv_decode_attn_update — one decode step of every row (VoxZip, second stage):
 *   append (k_t, v_t) at the row's free slot with pos = L + steps;
 *   p_g = softmax(q_{t,g} K^T / sqrt(d)) over the count + 1 entries;
 *   out_g = p_g V  (computed before eviction);
 *   A <- gamma * A + sum_g p_g  (the appended entry starts from 0);
 *   if count + 1 > b: evict the entry with the smallest A among the middle —
 *   not the T smallest positions (sinks), not the M largest (recent), ties
 *   evict the larger position — and its slot becomes the next free slot.
 *   q_t : device, [rows][g][d] dtype;  k_t, v_t : device, [rows][d] dtype.
 *   out : device, [rows][g][d] dtype.
 * bf16 caches with g <= 8: one persistent launch of one CTA per SM, whose
 * CTAs that share a row wait for each other (bounded: a wait that runs out
 * sets KV_DEV_TIMEOUT, and the decode state is then undefined until
 * kv_decode_init runs again). Steps on one stream are ordered; steps of one
 * cache must not overlap on different streams.
 * Errors: KV_ERR_ARG, KV_ERR_WORKSPACE, KV_ERR_CUDA.
 */
int kv_decode_attn_update(const kv_shape* shape, const int32_t* L, int32_t n_seq, const kv_params* params,
                          kv_cache* cache, const void* q_t, const void* k_t, const void* v_t, void* out,
                          void* stream);

/*
 * kv_score_noalloc — kv_score for callers that cannot allocate device memory
 * (no counterpart in the pages: a deployment variant of the same operation).
 * Same arguments, layout and result as kv_score, minus the workspace: the
 * scratch is a file-scope device array of KV_NOALLOC_SCRATCH_BYTES held by
 * every GPU that loads this library until the process exits.
 *   - Each call looks up the array's device address (cudaGetSymbolAddress);
 *     the first call on a device may load the library's device code there,
 *     so make that first call before any stream capture.
 *   - Batches whose scratch (kv_workspace_bytes) exceeds the limit return
 *     KV_ERR_WORKSPACE and launch nothing.
 *   - Every call shares the one array and it keeps the last call's contents;
 *     the status word is cleared by each call. Calls that overlap on the GPU
 *     (different streams, or different threads' streams) race on it: order
 *     them on one stream or synchronise between them.
 *   - Allocates nothing (no cudaMalloc/cudaFree, no allocating library call).
 *     Device-side errors (a bounded wait that ran out) go to the array's
 *     status word: read it with kv_score_noalloc_status.
 * Errors: as kv_score (KV_ERR_WORKSPACE when the batch is too large).
 */
#define KV_NOALLOC_SCRATCH_BYTES (8u << 20)
int kv_score_noalloc(const kv_shape* shape, const int32_t* L, int32_t n_seq, const void* qwin, const void* K,
                     float* s, void* stream);

/* The device status word (KV_DEV_* bits) of the last kv_score_noalloc call
 * on the current device, copied to *status_host after `stream` (synchronises
 * it; issue it on the scoring call's stream). Returns KV_OK, KV_ERR_ARG or
 * KV_ERR_CUDA. */
int kv_score_noalloc_status(int32_t* status_host, void* stream);

/* Time limit of the library's bounded device waits, in nanoseconds of the
 * GPU's global timer, for every launch made after the call (process-wide,
 * all devices); returns the previous limit. Default 2 000 000 000 (2 s).
 * A wait that runs out records KV_DEV_TIMEOUT in the call's status word; the
 * kernel lets its copies and tensor-core operations in flight finish (a drain
 * with a fixed limit of its own), releases its tensor memory and returns.
 * 0 makes every wait give up unless what it waits for has already happened,
 * which drives the timeout paths in tests. (No counterpart on the pages: a
 * safety limit of this implementation.) */
uint64_t kv_set_wait_limit_ns(uint64_t limit_ns);

/* Copies the device status word to the host (synchronises `stream`);
 * returns KV_OK or KV_ERR_CUDA. */
int kv_read_device_status(const int32_t* status_dev, int32_t* status_host, void* stream);

/*
 * Debug builds (libkvcomp_debug.so: the same sources compiled with
 * -DKV_DEBUG_CHECKS). Every kernel checks the indices it takes from data
 * (kept positions, slot numbers and slot ranges, cluster, node and member
 * ids, pooled row ranges, recalled blocks) against the extent of the
 * buffer or row they address; a failed check skips that access (and, where
 * the rest of the row depends on it, the row) and sets KV_DEV_BOUNDS in the
 * library's check word. Release builds compile the checks away.
 * kv_debug_checks returns 1 in a debug build and 0 in a release build.
 */
int kv_debug_checks(void);

/* The library's check word (KV_DEV_BOUNDS or 0; always 0 in a release
 * build) copied to *word_host after all earlier work on the current device
 * (synchronises the device); clear != 0 resets it to 0 afterwards.
 * Errors: KV_ERR_ARG (null word_host), KV_ERR_CUDA. */
int kv_debug_check_word(int32_t* word_host, int32_t clear);

/* Human-readable name of a status code. */
const char* kv_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* KVCOMP_H */
