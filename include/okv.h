/*
 * okv.h -- C ABI of the B200 INT2 KV-cache library (OSCAR-style rotations).
 *
 * What the library computes, as the pages describe it:
 *   - keys are rotated by R_K = U_K H P_br, with U_K the eigenbasis of the
 *     calibration query covariance; values by R_V = U_V H P_br, with U_V the
 *     eigenbasis of the attention-score-weighted value covariance; H is a
 *     normalised Hadamard and P_br the bit-reversal permutation, applied in
 *     that order (gen-hub.ru, "Together AI открывает OSCAR…", section
 *     "Что придумали в Together AI"; aiforradalom.hu, "Az Apple, a Google és
 *     a NYU új technikái…", section "OSCAR: figyelem-tudatos és bevetésre kész");
 *   - the rotated vectors are stored as 2-bit codes with a per-group scale
 *     and minimum (bigsaas.top, "Revolução no Serviço de LLMs…", section
 *     "Resultados e Métricas de Desempenho": INT2 at about 2.28 bits);
 *   - sink and recent tokens are also kept in 16-bit, older ones only in
 *     INT2, in a paged cache (encorp.ai, "KV cache compression е
 *     инфраструктурно решение…", section "OSCAR има значение…"; the pages
 *     give no sink count, so it is a cache parameter, num_sink, 0 by default;
 *     192 sinks with the 128-token window keep the ~0.24 % of a 128K context
 *     that section quotes);
 *   - decode attention reads that cache; decode is bound by reading the cache
 *     from HBM (aiforradalom.hu intro).
 *
 * Conventions
 *   - Row vectors: x_rot = x R.  Matrices are row-major fp32.
 *   - d (head_dim) = 128, 16 tokens per block, fp16 window W = 128 tokens;
 *     quantisation group g = 128 (one group per token-head), 64 or 32
 *     channels.  The groups are runs of consecutive channels after the
 *     rotation, so with g < 128 the bit-reversal permutation hands every
 *     group an even share of the importance order that U and H leave (the
 *     reason the pages give for P_br: gen-hub.ru "Что придумали в Together
 *     AI").  Effective bits per element: 2 + 32/g.  Other values return
 *     OKV_ERR_UNSUPPORTED.
 *   - "device" pointers point to memory of the current CUDA device; "host"
 *     pointers to ordinary host memory.  The caller owns every buffer; the
 *     library allocates nothing on the hot path and never synchronises the
 *     stream.  `stream` is a cudaStream_t (NULL = legacy default stream).
 *   - Every call validates its arguments on the host before launching and
 *     returns a status.  Launch failures return OKV_ERR_CUDA.  Conditions
 *     only the device can see (a block id outside [0, num_blocks), a position
 *     beyond the block table, a decode length beyond the table) are skipped by
 *     the kernels and recorded in `desc->status_word` (if not NULL) as a
 *     bitwise OR of OKV_DEV_* flags; the caller reads it when it chooses.
 *   - okv_last_error_string() describes the last non-OK status of the
 *     calling thread.
 *
 * Physical layout of one block (16 tokens) of one KV head, with ng = 128/g
 * groups per token: 1024 + 128 ng bytes (1152, 1280 or 1536 for g = 128, 64,
 * 32; okv_block_head_bytes)
 *   [   0,  512) K codes, token-major: 16 rows of 32 bytes; byte b of row t
 *                holds channels 4b..4b+3 of token t at bits 0-1, 2-3, 4-5, 6-7
 *                (channel = index after the rotation, i.e. after P_br).
 *   [ 512, 1024) V codes, the same bytes regrouped: 32 chunks of 16 bytes;
 *                byte b of token t sits at 512 + ((b>>2)*4 + (t>>2))*16
 *                + (b&3)*4 + (t&3).
 *   [1024, 1024 + 64 ng) K scale and min: token t, group k (channels
 *                k g .. k g + g - 1) at 1024 + 4 (t ng + k), fp16 scale then
 *                fp16 min.
 *   [1024 + 64 ng, 1024 + 128 ng) V scale and min, the same.
 * Block `blk`, head `h` starts at pages + (blk * num_kv_heads + h) *
 * okv_block_head_bytes(g).
 * Window ring: fp16 [num_seq_slots][num_kv_heads][2 (K,V)][W][d]; position p
 * of a sequence lives in row p % W; values are the rotated vector in fp16.
 * Sink rows: fp16 [num_seq_slots][num_kv_heads][2 (K,V)][num_sink][d];
 * position p < num_sink lives in row p.
 * Every position is quantised to INT2; decode of a sequence of length L reads
 * positions [0, min(S, L)) from the sink rows (S = num_sink),
 * [max(L - W, S), L) from the window ring and [S, L - W) from INT2 blocks.
 */
#ifndef OKV_H
#define OKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  OKV_OK = 0,
  OKV_ERR_INVALID_ARG = 1,  /* bad pointer, size, alignment or shape      */
  OKV_ERR_UNSUPPORTED = 2,  /* valid but not implemented (d != 128, ...)  */
  OKV_ERR_CUDA = 3,         /* a CUDA runtime call or a launch failed     */
  OKV_ERR_NUMERIC = 4,      /* the eigensolver did not converge, or a loaded
                               rotation is not orthogonal                 */
  OKV_ERR_IO = 5,           /* a file could not be opened, read or written,
                               or is not a valid rotations file           */
} okv_status;

/* bits of *status_word written by the kernels */
#define OKV_DEV_BAD_BLOCK 1u     /* block id outside [0, num_blocks)       */
#define OKV_DEV_BAD_POS 2u       /* position or length beyond the table    */
#define OKV_DEV_BAD_SLOT 4u      /* sequence slot outside [0, num_seq_slots) */
#define OKV_DEV_TIMEOUT 8u       /* a bulk copy did not land within ~1 s; the kernel gave up */

/* okv_append_quantize flags */
#define OKV_PRE_ROTATED 1u  /* k, v are fp32 values already in the rotated basis */

#define OKV_HEAD_DIM 128
#define OKV_BLOCK_TOKENS 16
#define OKV_WINDOW 128
#define OKV_MAX_SINK 1024
#define OKV_BLOCK_HEAD_BYTES 1152  /* bytes of one block-head with g = 128 */

typedef struct {
  int32_t num_q_heads;        /* Hq; a multiple of num_kv_heads            */
  int32_t num_kv_heads;       /* Hkv                                        */
  int32_t head_dim;           /* must be 128                                */
  int32_t group;              /* quantisation group: 128, 64 or 32 channels */
  int32_t block_tokens;       /* must be 16                                 */
  int32_t window;             /* must be 128                                */
  int32_t num_blocks;         /* physical blocks in `pages`                 */
  int32_t num_seq_slots;      /* sequences the window ring holds            */
  int32_t max_blocks_per_seq; /* row length of every block table            */
  int32_t num_sink;           /* sink tokens kept fp16: a multiple of 16 in
                                 [0, OKV_MAX_SINK], else OKV_ERR_UNSUPPORTED */
  void* pages;                /* device, num_blocks*Hkv*1152 B, 16-B aligned */
  void* window_ring;          /* device fp16, layout above, 16-B aligned     */
  const float* u_k;           /* device fp32 [Hkv][d][d]: U_K of each KV head */
  const float* u_v;           /* device fp32 [Hkv][d][d]: U_V of each KV head */
  uint32_t* status_word;      /* device, nullable: OKV_DEV_* flags (OR-ed)   */
  void* sink_rows;            /* device fp16, layout above, 16-B aligned;
                                 may be NULL when num_sink = 0             */
  void* r_image;              /* device, okv_r_image_bytes(Hkv) B, 16-B aligned,
                                 nullable: the prefill append's staged R of
                                 every (KV head, K|V), written by
                                 okv_build_r_image for the current u_k, u_v
                                 (rebuild it after changing them).  NULL: each
                                 prefill append stages R itself.           */
} okv_cache_desc;

/* Offline calibration of the rotations, on the host in fp64 (once per layer).
 * q: host fp32 [nq][hq][d] calibration queries; k, v: host fp32 [nk][hkv][d]
 * calibration keys and values.  Query head j belongs to KV head j/(hq/hkv).
 *   C_Q = mean of q q^T over the nq*G queries of the group (uncentred),
 *   C_S = sum_ij p_ij v_j v_j^T / sum_ij p_ij, p_ij = softmax_j(q_i.k_j/sqrt(d)),
 *   U = eigenvectors by descending eigenvalue, each column signed so that its
 *   largest-magnitude entry is positive; R = U H P_br.
 * Outputs (host fp32 [hkv][d][d], each nullable): r_k, r_v, u_k, u_v.
 * Errors: INVALID_ARG (null inputs, nq/nk < 1, hq % hkv), UNSUPPORTED
 * (d != 128), NUMERIC (Jacobi sweeps did not converge).
 * Pages: gen-hub.ru "Что придумали в Together AI" (both covariances and the
 * three-step transform) and "Открытый код — это серьёзно" (offline, once). */
okv_status okv_calibrate_rotations(const float* q, int64_t nq, const float* k, const float* v,
                                   int64_t nk, int32_t hq, int32_t hkv, int32_t d, float* r_k,
                                   float* r_v, float* u_k, float* u_v);

/* Rotation files: U_K and U_V of every layer and KV head of a model, so that a
 * deployment loads precomputed rotations instead of calibrating (gen-hub.ru,
 * "Открытый код — это серьёзно": rotations are computed offline, once per
 * model, and shipped; aiforradalom.hu, "OSCAR: figyelem-tudatos…": a set of
 * precomputed rotations per supported model).  The pages give no format; this
 * one is little-endian:
 *   32-byte header: "OKVROTS1", u32 version (1), u32 d, u32 num_layers,
 *   u32 num_kv_heads, u32 tag_len, u32 0;
 *   tag_len bytes of tag (free text, e.g. the model name; at most 4096);
 *   fp32 U_K [num_layers][num_kv_heads][d][d], fp32 U_V the same;
 *   u64 FNV-1a (64-bit) of everything before it.
 * Host buffers throughout; no CUDA call is made.
 * okv_save_rotations: tag may be NULL.  Errors: INVALID_ARG (NULL, empty
 *   shape, tag too long), UNSUPPORTED (d != 128), IO (open or write failed).
 * okv_rotations_file_shape: reads the header; each output is nullable.
 * okv_load_rotations: the shape must match the file's; tag (nullable)
 *   receives the tag, truncated to tag_capacity - 1 bytes and NUL-terminated;
 *   verify != 0 also checks max |U^T U - I| <= 1e-4 for every matrix.  Errors:
 *   INVALID_ARG (NULL, shape mismatch), UNSUPPORTED (other format version), IO
 *   (missing, truncated, trailing bytes, bad magic or checksum), NUMERIC
 *   (verify failed).  On IO and NUMERIC errors u_k and u_v may have been
 *   partly written. */
okv_status okv_save_rotations(const char* path, int32_t num_layers, int32_t num_kv_heads, int32_t d,
                              const float* u_k, const float* u_v, const char* tag);
okv_status okv_rotations_file_shape(const char* path, int32_t* num_layers, int32_t* num_kv_heads, int32_t* d,
                                    int32_t* tag_len);
okv_status okv_load_rotations(const char* path, int32_t num_layers, int32_t num_kv_heads, int32_t d, float* u_k,
                              float* u_v, char* tag, size_t tag_capacity, int32_t verify);

/* Bytes of one block-head (16 tokens of one KV head) for quantisation group
 * `group` (1152, 1280, 1536 for 128, 64, 32), 0 for an unsupported group.
 * The pages' INT2 format with a scale and a minimum per group (bigsaas.top,
 * "Revolução no Serviço de LLMs…", section "Resultados e Métricas de
 * Desempenho"). */
size_t okv_block_head_bytes(int32_t group);

/* Bytes of the optional staged-rotation buffer `r_image`: for every KV head,
 * K and V, R = U H P_br / sqrt(d) split into three bf16 parts (their sum is R
 * to about 2^-24 relative), 96 KB in the operand layout of the tcgen05 append. */
size_t okv_r_image_bytes(int32_t num_kv_heads);

/* Fill desc->r_image from desc->u_k and desc->u_v (one CTA per (KV head,
 * K|V), asynchronous on `stream`).  The prefill append then copies its R
 * instead of staging it from U at the start of every CTA.  Returns
 * OKV_ERR_INVALID_ARG when r_image is NULL or misaligned.  Pages: gen-hub.ru,
 * "Что придумали в Together AI" (R = U, then H, then P_br, precomputed once
 * per layer: aiforradalom.hu, "OSCAR: figyelem-tudatos és bevetésre kész"). */
okv_status okv_build_r_image(const okv_cache_desc* desc, void* stream);

/* Bytes the caller allocates for `pages`, `window_ring` and `sink_rows`. */
size_t okv_pages_bytes(int32_t num_blocks, int32_t num_kv_heads, int32_t group);
size_t okv_window_bytes(int32_t num_seq_slots, int32_t num_kv_heads);
size_t okv_sink_bytes(int32_t num_seq_slots, int32_t num_kv_heads, int32_t num_sink);

/* Append T tokens: rotate each K and V vector of every KV head by its R,
 * quantise it to 2-bit codes with fp16 scale and min (fp32 round-to-nearest
 * steps: s = fp16((max-min)/3), m = fp16(min), c = clamp(rint((z-m)/s),0,3),
 * c = 0 when s = 0; fp16 conversions saturate at +-65504), write codes and
 * (s, m) into slot pos%16 of block block_table[slot][pos/16], and, when
 * pos >= slot_lens[slot] - W, also write the fp16 rotated vector into the
 * window ring row pos % W, and when pos < num_sink into sink row pos.
 *   k, v: device [T][Hkv][d], bf16 (or fp32 already rotated with OKV_PRE_ROTATED);
 *   seq_slot, pos: device int32 [T]; block_table: device int32
 *   [num_seq_slots][max_blocks_per_seq]; slot_lens: device int32
 *   [num_seq_slots], each sequence's length after this append;
 *   rotated_out: device fp32 [T][2][Hkv][d] (nullable), the rotated fp32
 *   vectors the quantiser saw.
 * Tokens with equal (slot, pos) in one call race; T = 0 is a no-op.
 * Pages: gen-hub.ru "Что придумали в Together AI" (U, then H, then P_br);
 * bigsaas.top "Resultados e Métricas de Desempenho" (INT2). */
okv_status okv_append_quantize(const okv_cache_desc* desc, const void* k, const void* v, int32_t T,
                               const int32_t* seq_slot, const int32_t* pos,
                               const int32_t* block_table, const int32_t* slot_lens,
                               uint32_t flags, float* rotated_out, void* stream);

/* Workspace bytes okv_decode_attention (and okv_decode_step) needs for batch
 * B on the current device: the rotated queries in the forms the split-K
 * kernel reads, the cost prefix, and one fp32 partial (o', max, sum) per query
 * head for every split-K CTA and batch entry -- so it grows with the device's
 * SM count.  The split-K partials are the log-sum-exp pieces of the decode
 * attention that streams the cache from HBM (aiforradalom.hu, "Az Apple, a
 * Google és a NYU új technikái…", intro: decode is bound by reading the KV
 * cache).  Returns 0 for an invalid descriptor or B < 0. */
size_t okv_decode_workspace_bytes(const okv_cache_desc* desc, int32_t B);

/* Decode attention for one new query per sequence.
 *   q: device bf16 [B][Hq][d]; seq_slot: device int32 [B] (row of block table
 *   and window ring); block_table as above; context_lens: device int32 [B],
 *   tokens in the cache for each sequence (the caller appends the step's own
 *   token first); out: device fp32 [B][Hq][d]; workspace: device, at least
 *   okv_decode_workspace_bytes(desc, B) bytes, 256-B aligned.
 * Query head j reads KV head j/(Hq/Hkv).  With L = context_lens[b] and
 * S = num_sink, positions [0, min(S, L)) are read from the fp16 sink rows,
 * [S, L-W) from the INT2 blocks and [max(S, L-W), L) from the fp16 window;
 * q~ = q R_K, softmax(q~ x^T / sqrt(d)) over those, then o = o~ R_V^T.
 * L = 0 gives zeros.  Launches three kernels on `stream` (query rotation,
 * split-K attention, split combine with the value un-rotation).
 * Pages: aiforradalom.hu intro (decode streams the cache from HBM);
 * gen-hub.ru "Что придумали в Together AI" (rotations of Q and of SV). */
okv_status okv_decode_attention(const okv_cache_desc* desc, const void* q, int32_t B,
                                const int32_t* seq_slot, const int32_t* block_table,
                                const int32_t* context_lens, float* out, void* workspace,
                                size_t workspace_bytes, void* stream);

/* Size of the device array behind okv_decode_attention_noalloc (8 MiB).  A
 * batch fits when okv_decode_workspace_bytes(desc, B) is at most this, which
 * depends on the SM count: on a 148-SM B200, up to 57 sequences with 32 query
 * and 8 KV heads (so a 64-sequence batch is refused), up to 28 with 64 and 8. */
#define OKV_NOALLOC_SCRATCH_BYTES (8u << 20)

/* One decode step in one call: append this step's new tokens, then decode.
 * Equivalent to okv_append_quantize(desc, k, v, T, new_seq_slot, new_pos,
 * block_table, slot_lens, 0, NULL, stream) followed by
 * okv_decode_attention(desc, q, B, seq_slot, block_table, context_lens, out,
 * workspace, workspace_bytes, stream), with the same arguments, layouts,
 * ownership and errors as those two calls (K/V are bf16 here; there is no
 * pre-rotated form).  For T < 128 the append and the query rotation share one
 * launch, which saves a kernel's latency per step; longer runs take the
 * append's own tensor-core launch.  T = 0 decodes only; B = 0 appends only.
 * (The pages' append and decode steps: gen-hub.ru, "Что придумали в Together
 * AI"; encorp.ai, "OSCAR има значение…".) */
okv_status okv_decode_step(const okv_cache_desc* desc, const void* k, const void* v, int32_t T,
                           const int32_t* new_seq_slot, const int32_t* new_pos, const int32_t* slot_lens,
                           const void* q, int32_t B, const int32_t* seq_slot, const int32_t* block_table,
                           const int32_t* context_lens, float* out, void* workspace, size_t workspace_bytes,
                           void* stream);

/* Decode attention that allocates nothing and takes no workspace.  The pages
 * have no counterpart to this call: it exists for callers that cannot
 * allocate device memory -- a plugin handed only its tensors by an engine
 * that owns all device memory, or code that must not call cudaMalloc because
 * it can synchronise the device and stall other streams.
 *   Same arguments, results and kernels as okv_decode_attention, minus the
 *   workspace.  Scratch is a static device array of OKV_NOALLOC_SCRATCH_BYTES
 *   that every GPU which loads the library holds until process exit; a batch
 *   whose scratch (okv_decode_workspace_bytes) exceeds it is rejected with
 *   OKV_ERR_INVALID_ARG before anything runs.
 *   The first call on each device looks up the array's device address with
 *   that device current; make that first call before any stream capture.
 *   All calls share the one array (it keeps the last call's contents, none of
 *   which a later call relies on): calls that overlap on the GPU -- on
 *   different streams, or from different threads -- race and must be
 *   serialised by the caller. */
okv_status okv_decode_attention_noalloc(const okv_cache_desc* desc, const void* q, int32_t B,
                                        const int32_t* seq_slot, const int32_t* block_table,
                                        const int32_t* context_lens, float* out, void* stream);

/* Chunked-prefill attention over the cache, for one sequence.  The chunk's
 * T tokens must already be appended (okv_append_quantize), so sequence
 * `slot` holds context_len = L tokens and the chunk is positions L - T ..
 * L - 1.  Query i (position L - T + i) of head j attends to positions
 * 0 .. L - T + i of KV head j/(Hq/Hkv), causally, each read as the cache
 * holds it at length L: positions [0, min(S, L)) from the sink rows,
 * [max(L - W, S), L) from the window ring, the rest from INT2 blocks.  As in
 * decode, q~ = q R_K and o = softmax(q~ x^T / sqrt(d)) x_V R_V^T.
 *   q: device bf16 [T][Hq][d]; slot, context_len: host ints (T <= L <=
 *   max_blocks_per_seq * 16); block_table: device, as above; out: device
 *   fp32 [T][Hq][d]; workspace: device, at least
 *   okv_prefill_workspace_bytes(desc, T) bytes, 256-B aligned.
 * Three launches on `stream` (query rotation, attention on the tensor cores,
 * normalisation and value un-rotation).  Errors: INVALID_ARG (NULL, sizes,
 * slot or context_len out of range, workspace too small); block ids outside
 * [0, num_blocks) set OKV_DEV_BAD_BLOCK and those positions are skipped.
 * Pages: aiforradalom.hu, "Az Apple, a Google és a NYU új technikái…",
 * section "OSCAR: figyelem-tudatos és bevetésre kész", and gen-hub.ru
 * "Что это даёт на практике" (the compressed cache serves paged attention
 * and prefix caching, so a prefill chunk attends over the INT2 history);
 * gen-hub.ru "Что придумали в Together AI" (the rotations of Q and of SV). */
size_t okv_prefill_workspace_bytes(const okv_cache_desc* desc, int32_t T);
okv_status okv_prefill_attention(const okv_cache_desc* desc, const void* q, int32_t T, int32_t slot,
                                 int32_t context_len, const int32_t* block_table, float* out, void* workspace,
                                 size_t workspace_bytes, void* stream);

/* Gather and dequantise the cache into dense fp32 (the INT2 format's inverse:
 * s*c + m with the fp16 scale and minimum of each group; bigsaas.top,
 * "Revolução no Serviço de LLMs…", section "Resultados e Métricas de
 * Desempenho": INT2 values at about 2.28 bits; the original basis undoes
 * R = U H P_br, gen-hub.ru "Что придумали в Together AI").
 *   which: 0 keys, 1 values.  basis: 0 rotated (as stored), 1 original
 *   (multiplied back by R^T).  source: 0 INT2 for every position, 1 as decode
 *   reads it (fp16 for the last W positions and the first num_sink).  out: device fp32
 *   [B][Hkv][max_ctx][d]; rows at positions >= context_lens[b] are zero.
 * INT2 values are s*c + m computed with one fused multiply-add. */
okv_status okv_dequantize(const okv_cache_desc* desc, int32_t B, const int32_t* seq_slot,
                          const int32_t* block_table, const int32_t* context_lens,
                          int32_t max_ctx, int32_t which, int32_t basis, int32_t source,
                          float* out, void* stream);

/* Measurement hook: the next okv_decode_attention call made by this thread
 * records `start_event` just before its split-K attention kernel and
 * `stop_event` just after it (both cudaEvent_t, recorded on the call's
 * stream), then forgets them.  Passing two NULLs clears a pending request.
 * Lets a caller time the dominant kernel inside a running decode step.
 * Errors: INVALID_ARG if exactly one event is NULL. */
okv_status okv_time_next_decode_kernel(void* start_event, void* stop_event);

const char* okv_status_string(okv_status s);
const char* okv_last_error_string(void);
int32_t okv_version(void);

#ifdef __cplusplus
}
#endif
#endif /* OKV_H */
