/*
 * kvq.h -- C ABI of libkvq.so, the B200 (sm_100a) quantized KV-cache library.
 *
 * Two halves of one hot path:
 *   1. kvq_write: quantize bf16 K/V rows and scatter them into a preallocated
 *      cache by slot (int8 affine per token+head, or per-32 FP8 E4M3 /
 *      MX-FP8 / MX-FP4 blocks); kvq_sink_plan / kvq_sink_mask assign the slots
 *      and build the additive mask of an attention-sink / ring cache.
 *   2. kvq_decode_attn / kvq_prefill_attn: scaled dot-product attention that
 *      reads the int8 cache and dequantizes it in registers, with GQA, a
 *      kv_len bound read on the device, a per-tile causal bound and an
 *      additive mask.
 *
 * Conventions shared by every entry point
 *   - Pointers are DEVICE pointers (CUDA global memory of the current device)
 *     unless a parameter says "host".  The caller owns every buffer; the
 *     library never allocates, frees, or synchronizes the host.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  All work is enqueued asynchronously on it and no call reads
 *     device memory on the host: kvq_write, kvq_sink_plan, kvq_sink_mask,
 *     kvq_decode_attn and kvq_prefill_attn can be captured in a CUDA graph.
 *   - bf16 means IEEE binary16-brain (torch.bfloat16) bit patterns.
 *   - Return value: KVQ_OK (0) or a negative host status (below).  A non-zero
 *     status means nothing was enqueued, except KVQ_ECUDA from a failed launch.
 *   - Conditions only visible on the device never trap: the offending item is
 *     skipped (or clamped) and a KVQ_ERR_* bit is OR-ed into *err_word
 *     (nullable, int32 device word, never cleared by the library).
 *   - Calls that share output buffers must be ordered on streams by the caller.
 */
#ifndef KVQ_H
#define KVQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Host status codes. */
#define KVQ_OK 0
#define KVQ_EINVAL (-1)       /* null pointer, bad size, misaligned pointer, bad stride */
#define KVQ_EUNSUPPORTED (-2) /* a valid request this build does not implement */
#define KVQ_ECUDA (-3)        /* the CUDA launch itself failed */
#define KVQ_ESCRATCH (-4)     /* kvq_decode_attn_static: the problem needs more than the static scratch */

/* Device error-word bits (OR-ed into *err_word). */
#define KVQ_ERR_SLOT_RANGE 1   /* a slot outside [0, num_slots) other than -1 was skipped */
#define KVQ_ERR_KV_LEN_RANGE 2 /* *kv_len outside [0, S] (or [Lq, S] for prefill) was clamped */
#define KVQ_ERR_INPUT_POS 4    /* *input_pos < 0: the plan wrote -1 slots and kv_len 0 */
#define KVQ_ERR_TIMEOUT 8      /* a bounded wait inside a kernel gave up; its output is invalid */

/* Cache-write modes. */
/* kvq_write modes.  They number cache formats, not the IndexerQuantCache page's
 * quant_mode (参数说明: 0 MX-FP8, 1 Normal, 2 HiFloat8, 3 MX-FP4, with the cache
 * type a separate attribute).  The page's (quant_mode, cache type) maps to:
 *   (0, FLOAT8_E4M3FN) -> 2   (0, FLOAT8_E5M2) -> 5   (3, -) -> 3
 *   (1, FLOAT8_E4M3FN) -> 1   (1, FLOAT8_E5M2) -> 4   (1, INT8 as uint8) -> 6
 *   (2, HiFloat8): not built (the page names the format but does not define it).
 * Modes 0 and 7 are the int8 and 4-bit affine caches of the other pages. */
#define KVQ_MODE_INT8_AFFINE 0 /* int8 codes, f32 scale + int8 zero point per (token, head) */
#define KVQ_MODE_FP8_E4M3 1    /* E4M3 codes, f32 scale per 32 elements ("Normal") */
#define KVQ_MODE_MXFP8 2       /* E4M3 codes, E8M0 scale per 32 elements */
#define KVQ_MODE_MXFP4 3       /* E2M1 codes two per byte, E8M0 scale per 32 elements */
#define KVQ_MODE_FP8_E5M2 4    /* E5M2 codes, f32 scale per 32 elements ("Normal", FLOAT8_E5M2 cache) */
#define KVQ_MODE_MXFP8_E5M2 5  /* E5M2 codes, E8M0 scale per 32 elements (MX-FP8, FLOAT8_E5M2 cache) */
#define KVQ_MODE_INT8_SYM 6    /* int8 codes (two's complement in a uint8 cache), f32 scale per 32 ("Normal", UINT8) */
#define KVQ_MODE_INT4_AFFINE 7 /* TQ4: 4-bit codes two per byte, f32 scale + zero point 0..15 per (token, head) */

/* round_scale values of kvq_write (E8M0-scaled modes 2, 3, 5) */
#define KVQ_SCALE_FLOOR 0 /* the exponent of amax / Q_MAX as it stands */
#define KVQ_SCALE_CEIL 1  /* amax / Q_MAX rounded up to a power of two */
#define KVQ_SCALE_OCP 2   /* OCP MX v1.0: 2^(floor(log2 amax) - emax of the element format) */

/*
 * kvq_write -- quantize x and scatter it into the cache, in place.
 *
 * Defines: ExecuTorch PR 24473, Summary (int8 entries quantized per token and
 * head, affine asymmetric, float32 scale, int8 zero point, written through
 * update_cache_with_indices); IndexerQuantCache page, 功能说明 / 计算公式 /
 * 参数说明 / 约束说明 (per-block dynamic quantization scale_g = max|x_g| / Q_MAX,
 * q_i = round(x_i / scale_g); results and scales scattered to slot_mapping,
 * -1 skips the token; cache and scale updated in place; d % 32 == 0, d <= 8192);
 * ExecuTorch PR 20351 commit notes (a static scatter along the position dim,
 * capturable in a CUDA graph).
 *
 * x            bf16, element (b, h, t, i) at x[b*xs[0] + h*xs[1] + t*xs[2] + i];
 *              x_strides (host, 4 entries, in elements) with xs[3] implied 1.
 *              The row start of every (b, h, t) must be 16-byte aligned.
 * B, H, T, D   batch, heads, tokens per batch row, row length.
 * slot_mapping int32 [B*T]: cache slot of token (b, t) = slot_mapping[b*T + t];
 *              -1 skips it; any other value outside [0, num_slots) is skipped
 *              and sets KVQ_ERR_SLOT_RANGE.  Duplicate slots: undefined result.
 * num_slots    S, slots per (b, h) in the cache.
 * Cache layouts (row-major, contiguous, 16-byte aligned):
 *   mode 0: codes int8 [B, H, S, D]; scales float [B, H, S]; zero_points int8 [B, H, S]
 *   modes 1, 4, 6: codes u8 [B, H, S, D]; scales float [B, H, S, D/32]; zero_points NULL
 *   modes 2, 5: codes u8 [B, H, S, D]; scales u8 (E8M0) [B, H, S, D/32]
 *   mode 3: codes u8   [B, H, S, D/2] (element 2i in the low nibble); scales u8 (E8M0)
 *   mode 7 (TQ4): codes u8 [B, H, S, D/2] (element 2i in the low nibble); scales float
 *           [B, H, S]; zero_points [B, H, S] holding 0..15.  The 4-bit form of mode 0:
 *           scale = max((mx - mn)/15, FLT_EPSILON), zp = clamp(-rne(mn/scale), 0, 15),
 *           q = clamp(rne(x/scale) + zp, 0, 15) (ExecuTorch PR 20351, commit notes: the
 *           TQ4 cache is nibble-packed on the last dim and written along positions).
 *   With B = H = 1 the block modes are the IndexerQuantCache [num_slots, d] layout.
 *   Q_MAX: 448 (E4M3), 57344 (E5M2), 6 (E2M1), 127 (mode 6: q = rne(x / scale)
 *   clamped to [-127, 127], stored as its two's-complement byte).
 * round_scale  modes 2, 3 and 5 (the E8M0-scaled modes; IndexerQuantCache,
 *              参数说明, round_scale): how the scale becomes a power of two.
 *              KVQ_SCALE_CEIL (1, the default reading) rounds amax / Q_MAX up;
 *              KVQ_SCALE_FLOOR (0) takes its exponent as it stands (the largest
 *              power of two not above it); KVQ_SCALE_OCP (2) takes the OCP
 *              Microscaling v1.0 rule 2^(floor(log2 amax) - emax), emax 8
 *              (E4M3), 15 (E5M2), 2 (E2M1).  With FLOOR and OCP codes saturate
 *              at Q_MAX.  Other values: KVQ_EINVAL.  Ignored by the other modes.
 * Sizes: modes 0 and 7 need D in {64, 128, 256}; the other modes need D % 32 == 0 and
 * D <= 8192 (KVQ_EUNSUPPORTED otherwise).  B, H, T >= 0 (0 enqueues nothing).
 * The arithmetic is binary32 with one round-to-nearest-even per operation, in
 * a fixed order, so codes, scales and zero points are reproducible bit for bit.
 */
int kvq_write(int mode, int round_scale, const void *x, int B, int H, int T, int D,
              const int64_t *x_strides, const int32_t *slot_mapping, int64_t num_slots, void *codes,
              void *scales, int8_t *zero_points, int32_t *err_word, void *stream);

/*
 * kvq_write_kv -- kvq_write of a step's K and V in one launch.
 *
 * Defines: as kvq_write; the pages write the key and the value of each new
 * token through the same slot_mapping (ExecuTorch PR 24473, Summary: K and V
 * caches updated through update_cache_with_indices; IndexerQuantCache page,
 * 功能说明: the cache update in place at slot_mapping).  The K rows are
 * written exactly as kvq_write(mode, round_scale, k, ..., k_codes, k_scales,
 * k_zero_points) and the V rows as the same call on v; bit for bit the same.
 *
 * k, v         bf16 inputs of one shape [B, H, T, D], each with its own strides
 *              (k_strides, v_strides: host, 4 entries, as x_strides).
 * k_*, v_*     the two caches, each in the layout of `mode` (see kvq_write).
 * Other arguments, checks and errors as for kvq_write.  Both kvq_write and
 * kvq_write_kv launch as programmatic dependents of the kernel before them:
 * they may start while it drains and read nothing before it has completed.
 */
int kvq_write_kv(int mode, int round_scale, const void *k, const void *v, int B, int H, int T, int D,
                 const int64_t *k_strides, const int64_t *v_strides, const int32_t *slot_mapping,
                 int64_t num_slots, void *k_codes, void *k_scales, int8_t *k_zero_points, void *v_codes,
                 void *v_scales, int8_t *v_zero_points, int32_t *err_word, void *stream);

/*
 * kvq_sink_plan -- slots of an attention-sink / ring cache for T new tokens.
 *
 * Defines: ExecuTorch PR 24473, Summary (CachePositionsManagerWithSink: a
 * pinned sink prefix plus a ring; the ring cache is the case sink_size = 0).
 * Position p = *input_pos + t goes to slot p if p < sink_size, else to
 * sink_size + (p - sink_size) mod (S - sink_size).
 *
 * input_pos    int32 device scalar, first position of the T tokens.
 * B, T         batch rows (all at the same positions) and tokens.
 * sink_size    pinned prefix length, 0 <= sink_size < S.
 * S            cache slots; T must be <= S - sink_size (else KVQ_EUNSUPPORTED).
 * slot_mapping int32 [B*T] out: the slot of token (b, t), ready for kvq_write.
 * slot_pos     int32 [S] in/out: the position each slot holds, -1 = empty.
 *              Initialise it to -1 once per sequence.
 * kv_len       int32 device scalar out: min(*input_pos + T, S), the attention bound.
 * *input_pos < 0 writes -1 slots and kv_len 0 and sets KVQ_ERR_INPUT_POS.
 */
int kvq_sink_plan(const int32_t *input_pos, int B, int T, int sink_size, int64_t S,
                  int32_t *slot_mapping, int32_t *slot_pos, int32_t *kv_len, int32_t *err_word,
                  void *stream);

/*
 * kvq_sink_mask -- additive float mask of an attention-sink / ring cache.
 *
 * Defines: ExecuTorch PR 24473, Summary (_create_causal_mask_for_attention_sink;
 * ring and sink caches use an additive float mask).  Query row r sits at
 * position *input_pos + r and sees slot s iff 0 <= slot_pos[s] <= *input_pos + r:
 * mask[r*S + s] = 0.0f if visible, -INFINITY otherwise.  Call it after the
 * kvq_sink_plan of the same tokens.
 *
 * input_pos  int32 device scalar.   Lq  query rows (>= 1).
 * slot_pos   int32 [S] from kvq_sink_plan.   mask  float [Lq, S] out.
 */
int kvq_sink_mask(const int32_t *input_pos, int Lq, const int32_t *slot_pos, int64_t S, float *mask,
                  void *stream);

/*
 * kvq_sink_plan_rows -- kvq_sink_plan for a batch whose rows sit at their own
 * positions (a ragged sink / ring batch).
 *
 * Defines: ExecuTorch PR 24473, Summary (CachePositionsManagerWithSink), read
 * per batch row: each row is its own sequence with its own position and its
 * own cache rows, so each keeps its own slot table.  Row b's token t at
 * position p = input_pos[b] + t goes to slot p if p < sink_size, else to
 * sink_size + (p - sink_size) mod (S - sink_size), of row b's cache.
 *
 * input_pos    int32 [B] device array, the first position of each row's T tokens.
 * slot_mapping int32 [B*T] out: the slot (within row b) of token (b, t), as
 *              kvq_write expects for a cache [B, H, S, ...].
 * slot_pos     int32 [B, S] in/out: per row, the position each slot holds,
 *              -1 = empty; initialise a row to -1 when its sequence starts.
 * kv_lens      int32 [B] out: min(input_pos[b] + T, S), for the _varlen
 *              attention entry points.
 * A row with input_pos[b] < 0 gets -1 slots and kv_lens[b] = 0 and sets
 * KVQ_ERR_INPUT_POS.  Sizes and checks as for kvq_sink_plan, and B <= 65535.
 */
int kvq_sink_plan_rows(const int32_t *input_pos, int B, int T, int sink_size, int64_t S, int32_t *slot_mapping,
                       int32_t *slot_pos, int32_t *kv_lens, int32_t *err_word, void *stream);

/*
 * kvq_sink_mask_rows -- kvq_sink_mask per batch row.
 *
 * Defines: as kvq_sink_mask (ExecuTorch PR 24473, Summary), per row: query row
 * r of batch row b sits at input_pos[b] + r and sees slot s iff
 * 0 <= slot_pos[b, s] <= input_pos[b] + r; mask[(b * Lq + r) * S + s] = 0.0f
 * if visible, -INFINITY otherwise.  input_pos int32 [B], slot_pos int32 [B, S],
 * mask float [B, Lq, S] (pass mask_batch_stride = Lq * S to the _varlen
 * attention).  S % 4 == 0; slot_pos and mask 16-byte aligned.
 */
int kvq_sink_mask_rows(const int32_t *input_pos, int B, int Lq, const int32_t *slot_pos, int64_t S, float *mask,
                       void *stream);

/*
 * kvq_decode_workspace_bytes -- size of the kvq_decode_attn workspace.
 *
 * Returns the bytes the split-K decode needs for (B, Hq, Hkv, D, S) on the
 * current device, or 0 for arguments kvq_decode_attn would reject.  The size
 * depends only on D, the q heads per kv head and the device's SM count (not
 * on B, Hkv or S).  Layout: the first 1 KiB holds 256 int32 merge counters,
 * at that offset for every shape; the per-CTA partial records follow.
 * Reuse rule: zero-fill the workspace once before its first use
 * (cudaMemsetAsync).  Every call that completes leaves the counters at zero,
 * and no call writes anything else into the first 1 KiB, so one workspace of
 * at least the size each call needs serves any sequence of calls, of any
 * shapes, ordered on streams, without clearing.  Two calls whose kernels run
 * at the same time must not share it.  After a call that set
 * KVQ_ERR_TIMEOUT, zero it again.
 */
size_t kvq_decode_workspace_bytes(int B, int Hq, int Hkv, int D, int64_t S);

/*
 * kvq_decode_attn -- one-query attention over the int8 cache (split-K).
 *
 * Defines: abaddon 0.2.0-rc.1 src/attention_cache/mod.rs, trait KvCache
 * (forward_attention: q [batch, num_heads, q_len, head_dim], GQA over
 * num_kv_heads, scale typically 1/sqrt(head_dim); a fused kernel that does not
 * materialise K/V); ExecuTorch PR 20351 commit notes (kv_len is an int32 GPU
 * scalar read on the device, no host sync, bounding the loop to the filled
 * length); ExecuTorch PR 24473, Summary (ring / sink caches add a float mask).
 *
 *   out[b, h, :] = softmax_j(sm_scale * q[b,h,:] . K[b,hk,j,:] + mask[j]) V[b,hk,j,:]
 *   over j in [0, *kv_len), hk = h / (Hq / Hkv),
 *   K[b,hk,j,d] = (k[b,hk,j,d] - k_zp[b,hk,j]) * k_scale[b,hk,j] (same for V).
 *
 * q            bf16 [B, Hq, 1, D] contiguous.   out  bf16 [B, Hq, 1, D] contiguous.
 * k, v         int8 [B, Hkv, S, D];  k_scale, v_scale float [B, Hkv, S];
 *              k_zp, v_zp int8 [B, Hkv, S] (the kvq_write mode-0 layout).
 * kv_len       int32 device scalar; values outside [0, S] are clamped and set
 *              KVQ_ERR_KV_LEN_RANGE.  kv_len 0 gives zeros.
 * mask         nullable float [S] (row 0 of an [Lq, S] mask), added to the
 *              scaled scores; -INFINITY hides a slot.  A row that sees no slot
 *              outputs zeros.
 * workspace    device buffer of workspace_bytes >= kvq_decode_workspace_bytes(),
 *              zero-filled before its first use (see above).
 * Launches one kernel on `stream`, as a programmatic dependent launch: it may
 * start while the kernel before it drains, and reads nothing before that kernel
 * has completed.  The CTA that completes a split (b, kv head) merges its
 * partials in CTA order, so results do not depend on timing.
 * Sizes: D in {64, 128, 256}; Hq % Hkv == 0; S % 16 == 0; every pointer
 * 16-byte aligned.
 */
int kvq_decode_attn(const void *q, int B, int Hq, int Hkv, int D, const int8_t *k, const float *k_scale,
                    const int8_t *k_zp, const int8_t *v, const float *v_scale, const int8_t *v_zp,
                    int64_t S, const int32_t *kv_len, const float *mask, float sm_scale, void *out,
                    void *workspace, size_t workspace_bytes, int32_t *err_word, void *stream);

/*
 * kvq_decode_attn_varlen -- kvq_decode_attn with one kv_len per batch row.
 *
 * Defines: as kvq_decode_attn; the device-side bound of ExecuTorch PR 20351
 * (commit notes: kv_len read on the device, bounding the loop to the filled
 * length) taken per batch row, so rows of a decode batch can hold different
 * context lengths.
 *
 * kv_lens      int32 [B] device array: row b attends over slots [0, kv_lens[b]).
 *              Values outside [0, S] are clamped and set KVQ_ERR_KV_LEN_RANGE;
 *              a row with kv_lens[b] = 0 outputs zeros.
 * mask         nullable float: row b adds mask[b * mask_batch_stride + s] to the
 *              score of slot s (a ragged sink / ring batch: kvq_sink_mask_rows
 *              with Lq = 1 writes it with stride S).
 * mask_batch_stride  floats between two rows' masks; 0 shares one mask [S]
 *              among all rows.  A multiple of 4 (KVQ_EINVAL otherwise); the
 *              mask holds (B - 1) * mask_batch_stride + S floats.
 * Other arguments, sizes and the workspace as for kvq_decode_attn.  Batches of
 * up to 1024 rows are cut into split units by each row's own length (rows of
 * kv_lens 0 own no work); larger batches are cut as for the longest row, and
 * tiles past a row's own length move no bytes.  With at most 32 rows of
 * different lengths each row's (kv head, head chunk) units may instead get CTAs
 * of their own, more for longer rows, when that costs no rounds of tiles; rows
 * of equal length are cut exactly as kvq_decode_attn cuts them (equal results).
 */
int kvq_decode_attn_varlen(const void *q, int B, int Hq, int Hkv, int D, const int8_t *k, const float *k_scale,
                           const int8_t *k_zp, const int8_t *v, const float *v_scale, const int8_t *v_zp,
                           int64_t S, const int32_t *kv_lens, const float *mask, int64_t mask_batch_stride,
                           float sm_scale, void *out, void *workspace, size_t workspace_bytes,
                           int32_t *err_word, void *stream);

/*
 * kvq_decode_attn_tq4 -- kvq_decode_attn over a TQ4 cache (kvq_write mode 7).
 *
 * Defines: as kvq_decode_attn, over the cache ExecuTorch PR 20351 (commit
 * notes) calls TQ4: nibble-packed on the last dim, D/2 bytes per slot, which
 * halves the decode's bytes again.  K = (k - k_zp) * k_scale with k a 4-bit
 * code 0..15 (element 2i in the low nibble of byte i), V likewise.
 *
 * k, v         u8 [B, Hkv, S, D/2];  k_scale, v_scale float [B, Hkv, S];
 *              k_zp, v_zp u8 [B, Hkv, S] holding 0..15.
 * Other arguments, sizes and the workspace as for kvq_decode_attn.  At D = 128
 * and 256 the kernel is kvq_decode_attn's on the tensor cores (codes unpacked to
 * bytes for q.K, to the fp16 values 1024 + c for P.V; exact); at D = 64 a
 * CUDA-core form of it (dp2a for q.k, packed fp32 FMA for p.v).
 */
int kvq_decode_attn_tq4(const void *q, int B, int Hq, int Hkv, int D, const uint8_t *k, const float *k_scale,
                        const uint8_t *k_zp, const uint8_t *v, const float *v_scale, const uint8_t *v_zp,
                        int64_t S, const int32_t *kv_len, const float *mask, float sm_scale, void *out,
                        void *workspace, size_t workspace_bytes, int32_t *err_word, void *stream);

/*
 * kvq_decode_block_workspace_bytes -- size of the kvq_decode_attn_block workspace
 * for (B, Hq, Hkv, D, S) on the current device; 0 for sizes it rejects.  The
 * workspace must be zero-filled before its first use (its first 1 KiB holds
 * merge counters, which every completed call leaves at zero, as for
 * kvq_decode_attn); it can then serve later calls of any shape that fit it.
 */
size_t kvq_decode_block_workspace_bytes(int B, int Hq, int Hkv, int D, int64_t S);

/*
 * kvq_decode_attn_block -- one-query attention over a per-32 block cache
 * (kvq_write modes 1-6).
 *
 * Defines: the attention of kvq_decode_attn, with K and V read from the
 * IndexerQuantCache block format (计算公式: x ~ code * scale_g, one scale per 32
 * elements along the head dim): E4M3 / E5M2 / int8 codes with float scales
 * (modes 1, 4, 6), E4M3 / E5M2 codes with E8M0 scales (modes 2, 5), E2M1 codes
 * two per byte with E8M0 scales (mode 3).
 *
 * mode         1..6, the kvq_write mode that wrote the cache.
 * k_codes, v_codes  u8 [B, Hkv, S, D] (mode 3: [B, Hkv, S, D/2]).
 * k_scales, v_scales  [B, Hkv, S, D/32]: float (modes 1, 4, 6) or E8M0 bytes.
 * kv_len, mask, q, out, sm_scale, err_word as for kvq_decode_attn.
 * workspace    device buffer of at least kvq_decode_block_workspace_bytes(),
 *              zero-filled before its first use.
 * Modes 1, 2, 4, 5, 6, and mode 3 at D >= 128, launch one kernel on `stream`:
 * the split decode of kvq_decode_attn on the tensor cores (TMA tiles, in-kernel
 * merge), with the codes converted to fp16 and multiplied by their group scale
 * over one power of two per slot (exact for E8M0 scales; one fp16 rounding per
 * element for float scales), that power of two applied to the fp32 score (K) or
 * to P (V).  Mode 3 at D = 64 launches two kernels (a CUDA-core split
 * attention, a merge).
 * Sizes: D in {64, 128, 256}; Hq % Hkv == 0 with Hq / Hkv <= 8; S % 16 == 0.
 * q, the codes, the scales, out and the mask 16-byte aligned.
 */
int kvq_decode_attn_block(int mode, const void *q, int B, int Hq, int Hkv, int D, const uint8_t *k_codes,
                          const void *k_scales, const uint8_t *v_codes, const void *v_scales, int64_t S,
                          const int32_t *kv_len, const float *mask, float sm_scale, void *out, void *workspace,
                          size_t workspace_bytes, int32_t *err_word, void *stream);

/*
 * kvq_prefill_attn -- Lq-query (chunked prefill) attention over the int8 cache.
 *
 * Defines: as kvq_decode_attn, plus ExecuTorch PR 20351 commit notes (the
 * chunk's rows sit at positions kv_len - Lq + i; with a causal mask row i sees
 * j <= kv_len - Lq + i; mask_is_causal enables the per-tile causal upper bound
 * loop_end = min(kv_len, (kv_len - Lq) + max(seq_pos in tile) + 1), which skips
 * KV tiles that are fully masked).  With is_causal the output is bit-identical
 * with or without the bound; with a causal additive mask alone it can differ in
 * a rare last bit (the fp16 P exponent then also sees the slots the mask hides).
 *
 * q, out        bf16 [B, Hq, Lq, D] contiguous.  Cache arguments as for decode.
 * kv_len        int32 device scalar, clamped to [Lq, S] (KVQ_ERR_KV_LEN_RANGE).
 * mask          nullable float [Lq, S] additive (row stride S).
 * is_causal     1: apply the causal rule above (full-context cache).
 * mask_is_causal 1: the caller asserts the combined mask is causal in slot
 *               order (is_causal, or a mask that hides j > kv_len - Lq + i),
 *               which enables the per-tile bound.
 * Sizes: D in {64, 128, 256}; Hq % Hkv == 0; S % 16 == 0; 1 <= Lq <= S.
 * Launches one kernel on `stream`: 128 query rows per CTA on the tcgen05
 * tensor cores, S = Q K^T and O += P V with fp16 operands and fp32
 * accumulation in tensor memory.  When the row blocks would leave most SMs
 * idle, a thread-block cluster of up to 4 CTAs shares each row block, each CTA
 * taking a share of its KV tiles; the shares merge through distributed shared
 * memory (no workspace).  K/V codes enter as the exact fp16 values
 * (c - zp); q enters as fp16 after one power-of-two rescale per CTA (exact for
 * every element at least 2^-32 times the CTA's largest |q|); k_scale multiplies the fp32
 * scores, and v_scale is folded into P = p * v_scale * 2^-E, rounded to fp16
 * once (relative error <= 2^-11).
 */
int kvq_prefill_attn(const void *q, int B, int Hq, int Hkv, int Lq, int D, const int8_t *k,
                     const float *k_scale, const int8_t *k_zp, const int8_t *v, const float *v_scale,
                     const int8_t *v_zp, int64_t S, const int32_t *kv_len, const float *mask,
                     int is_causal, int mask_is_causal, float sm_scale, void *out, int32_t *err_word,
                     void *stream);

/*
 * kvq_prefill_attn_varlen -- kvq_prefill_attn with one kv_len per batch row.
 *
 * Defines: as kvq_prefill_attn, with the chunk of batch row b at positions
 * kv_lens[b] - Lq + i (ExecuTorch PR 20351, commit notes, per row).
 *
 * kv_lens      int32 [B] device array, each clamped to [Lq, S]
 *              (KVQ_ERR_KV_LEN_RANGE).
 * mask         nullable float: query row i of batch row b adds
 *              mask[b * mask_batch_stride + i * S + s] to the score of slot s
 *              (kvq_sink_mask_rows writes it with stride Lq * S).
 * mask_batch_stride  floats between two batch rows' masks; 0 shares one mask
 *              [Lq, S] among all rows.  A multiple of 4 (KVQ_EINVAL otherwise).
 * Other arguments as for kvq_prefill_attn.
 */
int kvq_prefill_attn_varlen(const void *q, int B, int Hq, int Hkv, int Lq, int D, const int8_t *k,
                            const float *k_scale, const int8_t *k_zp, const int8_t *v, const float *v_scale,
                            const int8_t *v_zp, int64_t S, const int32_t *kv_lens, const float *mask,
                            int64_t mask_batch_stride, int is_causal, int mask_is_causal, float sm_scale, void *out,
                            int32_t *err_word, void *stream);

/*
 * kvq_prefill_attn_block -- Lq-query (chunked prefill) attention over a per-32
 * block cache (kvq_write modes 1-6).
 *
 * Defines: the attention of kvq_prefill_attn (positions, causal rule, per-tile
 * bound, additive mask), with K and V read from the IndexerQuantCache block
 * format (计算公式: x ~ code * scale_g, one scale per 32 elements along the
 * head dim), as for kvq_decode_attn_block.
 *
 * mode         1..6, the kvq_write mode that wrote the cache.
 * k_codes, v_codes  u8 [B, Hkv, S, D] (mode 3: [B, Hkv, S, D/2]).
 * k_scales, v_scales  [B, Hkv, S, D/32]: float (modes 1, 4, 6) or E8M0 bytes
 *              (modes 2, 3, 5; 0xFF, which kvq_write never stores, gives
 *              undefined results).
 * q, out, kv_len, mask, is_causal, mask_is_causal, sm_scale, err_word as for
 * kvq_prefill_attn.  No workspace.
 * Launches one kernel on `stream`, the tcgen05 kernel of kvq_prefill_attn.  Its
 * converters apply the scales per element: each slot's K (and V) is divided by
 * the power of two 2^E at or above its largest group scale and rounded to fp16,
 * and 2^E multiplies the fp32 scores (for V: folds into P).  E8M0 modes are
 * exact except for elements below 2^-24 of their slot's largest group factor;
 * float-scale modes round each element once (relative error <= 2^-11).
 * Sizes: D in {64, 128, 256}; Hq % Hkv == 0; S % 16 == 0; 1 <= Lq <= S; every
 * pointer 16-byte aligned.
 */
int kvq_prefill_attn_block(int mode, const void *q, int B, int Hq, int Hkv, int Lq, int D,
                           const uint8_t *k_codes, const void *k_scales, const uint8_t *v_codes,
                           const void *v_scales, int64_t S, const int32_t *kv_len, const float *mask,
                           int is_causal, int mask_is_causal, float sm_scale, void *out, int32_t *err_word,
                           void *stream);

/*
 * kvq_decode_attn_static -- kvq_decode_attn without a caller-supplied workspace.
 *
 * The pages have no counterpart of this entry point; it exists for callers
 * that cannot allocate device memory when they run attention: runtimes that
 * plan and own every byte of device memory up front, plain C hosts that have
 * no device allocator, and callers that must not let an allocation (and the
 * synchronisation cudaMalloc can imply) into their decode loop.  Instead of
 * the workspace it uses a buffer of KVQ_STATIC_SCRATCH_BYTES that lives in
 * the library itself (a file-scope __device__ array: every GPU that loads the
 * library holds it until the process exits).  It allocates nothing and frees
 * nothing.
 *
 * Arguments, layouts and results are those of kvq_decode_attn.  A problem
 * whose partial results would not fit the buffer (kvq_decode_workspace_bytes
 * above KVQ_STATIC_SCRATCH_BYTES) returns KVQ_ESCRATCH and enqueues nothing.
 * The first call on a device looks up the buffer's device address (with that
 * device current); make that first call before capturing a stream into a CUDA
 * graph.  All calls on a device share the one buffer: it starts zeroed, every
 * call that completes leaves its merge counters at zero, and the counters sit
 * at the same offset for every shape, so calls of different shapes can follow
 * one another in stream order.  Two calls whose kernels overlap on the GPU
 * (different streams without ordering) race on it and produce wrong results.
 * After a call that set KVQ_ERR_TIMEOUT, kvq_decode_static_reset() clears the
 * buffer.  A problem needs 1 KiB + 2 x SMs x HC x (D + 2) x 4 bytes, HC being
 * the largest divisor of Hq / Hkv not above 8: on a 148-SM B200 every D = 64
 * problem fits, D = 128 fits up to HC = 6 and D = 256 up to HC = 3; larger
 * ones return KVQ_ESCRATCH.
 */
#define KVQ_STATIC_SCRATCH_BYTES (1u << 20) /* 1 MiB per device */
int kvq_decode_attn_static(const void *q, int B, int Hq, int Hkv, int D, const int8_t *k,
                           const float *k_scale, const int8_t *k_zp, const int8_t *v,
                           const float *v_scale, const int8_t *v_zp, int64_t S, const int32_t *kv_len,
                           const float *mask, float sm_scale, void *out, int32_t *err_word,
                           void *stream);

/*
 * kvq_decode_static_reset -- zero the buffer of kvq_decode_attn_static on the
 * current device (one memset on `stream`).  Needed only after a call that set
 * KVQ_ERR_TIMEOUT, which can leave merge counters behind.
 */
int kvq_decode_static_reset(void *stream);

/*
 * kvq_set_wait_limit_ns -- bound on each main-loop wait of the decode kernels
 * (kvq_decode_attn, _varlen, _tq4, _static) and the prefill kernels
 * (kvq_prefill_attn, _varlen, _block).
 *
 * Every wait inside the library's kernels is bounded; a wait that runs out
 * sets KVQ_ERR_TIMEOUT in *err_word, the kernel stops issuing copies and
 * tensor-core work, waits (with the full 1 s bound, whatever this setting) for
 * what it already issued, completes its merge bookkeeping and returns (its
 * output is invalid; decode merge counters end at zero all the same).  The
 * default bound is 1 s; `ns` = 0 restores it.  The setting is process-wide and
 * applies to kernels launched after the call (a CUDA graph keeps the value it
 * captured).
 * A bound below 1000 ns gives up every main-loop wait at once, without
 * looking at the copy it waits for: that is how tests run the timeout path
 * deterministically, without withholding any copy.  Returns KVQ_OK.
 */
int kvq_set_wait_limit_ns(uint64_t ns);

/* A static, human-readable name for a host status code. */
const char *kvq_strerror(int status);

/* Library ABI version (major * 10000 + minor * 100 + patch). */
int kvq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KVQ_H */
