/*
 * kvcomp_next.h — calls of libkvcomp.so beyond the compression path of
 * kvcomp.h, on the same conventions (caller-owned device buffers, no
 * allocation, asynchronous on `stream`, status codes of kvcomp.h):
 *
 *   kv_voxzip_pool -> VoxZip first stage: semantic-anchored pooling of the
 *        audio feature rows ("VoxZip: Semantic-Anchored Temporal KV Cache
 *        Compression for Long-Context Audio Inference", 方法概述和架构,
 *        first stage, steps one to three).
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
 *   status     device int32 or NULL: KV_DEV_RANGE is OR-ed in (see above).
 * E_A, E_T and E_comp must not overlap. Errors: KV_ERR_ARG, KV_ERR_CUDA.
 */
int kv_voxzip_pool(const int32_t* L_a, int32_t n_seq, const double* tau_total, const int32_t* seg_off, int32_t d,
                   int32_t dtype, float conf_min, const kv_asr_segment* segs, const void* E_A, const void* E_T,
                   int64_t n_text_rows, void* E_comp, int32_t* src, int32_t* out_len, int32_t* status,
                   void* stream);

#ifdef __cplusplus
}
#endif

#endif /* KVCOMP_NEXT_H */
