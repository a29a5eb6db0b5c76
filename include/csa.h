/*
 * csa.h -- C ABI of libcsa.so: the CSA/HCA hybrid attention-layer core on one
 * NVIDIA B200 (sm_100a).
 *
 * The operations restate the attention layer of DeepSeek-V4 as described on
 * the page "DeepSeek-V4：迈向高效百万 Token 上下文智能" (a summary/translation of
 * the DeepSeek-V4 report), §3.3 "CSA 与 HCA 混合注意力", and on the page
 * "DeepSeek V4 完整技术报告", section "混合注意力：CSA + HCA":
 *   - csa_compress / hca_compress: softmax-gated compression of per-token KV
 *     into compressed entries (CSA: two overlapping groups, rate 1/m; HCA: one
 *     group, rate 1/m'), followed by RMSNorm and partial RoPE;
 *   - indexer_scores_topk: the lightning-indexer score
 *     I[t,s] = sum_h w[t,h] ReLU(q_I[t,h] . K_I[s]) and a causal per-query top-k;
 *   - sparse_mqa_attn / dense_hca_attn: multi-query attention in which each
 *     compressed entry is both key and value, over the selected entries (CSA)
 *     or all visible entries (HCA), plus a sliding window of per-token rows and
 *     a per-head sink logit, with RMSNorm + RoPE on the query and the output
 *     rotated back by the query position.
 *
 * Conventions for every call:
 *   - All tensor pointers are DEVICE pointers, row-major and contiguous, owned
 *     by the caller; the library allocates nothing.  Tensors must start on a
 *     16-byte boundary.
 *   - Calls are asynchronous on `stream` (a cudaStream_t passed as void*;
 *     NULL = the legacy default stream) and are stateless and reentrant.
 *   - Host-side validation runs before any launch and returns CSA_E_ARG or
 *     CSA_E_UNSUPPORTED without touching device memory.
 *   - Errors detected by a kernel (a bounded wait that expired, an index out of
 *     range, a logit beyond the static softmax bound) are written to a status
 *     word at the start of the workspace; csa_check_status() reads and clears
 *     it.  Kernels never trap.
 *   - Positions: token j of a prefill sequence sits at pos0 + j; compressed
 *     entry s covers tokens [m s, m s + m) counted from the start of the
 *     sequence and is visible to a query at position p iff s < floor((p+1)/m).
 *   - Stored entries and window rows are the TRANSFORMED rows (RMSNorm'd and
 *     rotated at their own positions), as a KV cache holds them; queries are
 *     raw and are normalised and rotated inside the attention calls.
 */
#ifndef CSA_H_
#define CSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ---------------------------------------------------- */
typedef int32_t csa_status;
#define CSA_OK 0
#define CSA_E_ARG 1          /* null pointer, negative size, misalignment, bad enum */
#define CSA_E_UNSUPPORTED 2  /* well-formed but outside what the kernels implement */
#define CSA_E_CUDA 3         /* a CUDA runtime call or kernel launch failed */
#define CSA_E_DEVICE 4       /* a kernel reported an error in the status word */
#define CSA_E_WORKSPACE 5    /* workspace missing or smaller than required */

/* device status-word codes (the `detail` of csa_check_status) */
#define CSA_DEV_OK 0u
#define CSA_DEV_TIMEOUT 1u     /* a bounded mbarrier wait ran out; results invalid */
#define CSA_DEV_RANGE 2u       /* a logit exceeded the static softmax bound (un-normalised keys) */
#define CSA_DEV_BAD_INDEX 3u   /* an index outside [-1, N) was skipped */
#define CSA_DEV_STREAM 4u      /* a stream state was invalid (sequence skipped) or its entry
                                  cache full (entry dropped); detail: the sequence */

/* ---- element types and flags ---------------------------------------- */
#define CSA_F32 0   /* float32 tensors, float32 arithmetic (CUDA cores) */
#define CSA_BF16 1  /* bfloat16 tensors, float32 accumulation (tensor cores where dense) */

#define CSA_F_NO_NORM 1u   /* skip RMSNorm (test hook) */
#define CSA_F_NO_ROPE 2u   /* skip RoPE and the output rotation (test hook) */
#define CSA_F_PORTABLE 4u  /* attention: use the CUDA-core kernel even for bf16 (cross-checks) */
#define CSA_F_MIXED 8u     /* attention: `entries` holds mixed BF16 / MX-FP8 records
                              (csa_store_mixed) instead of dtype rows */

/* Entry format shared by all calls.  c: entry / head dim (c/vec a power of two,
 * vec = 8 for bf16, 4 for f32); rope_dims: r, even, <= c, RoPE on dims
 * [c-r, c) in interleaved pairs (c-r+2i, c-r+2i+1) with angle
 * pos * rope_base^(-2i/r); norm_eps: RMSNorm epsilon (unit gain). */
typedef struct csa_fmt {
  int32_t c;
  int32_t rope_dims;
  float rope_base;
  float norm_eps;
  uint32_t flags;
} csa_fmt;

/* Workspace ops for csa_workspace_bytes(). */
#define CSA_OP_INDEXER 1
#define CSA_OP_SPARSE_ATTN 2
#define CSA_OP_DENSE_ATTN 3
#define CSA_OP_COMPRESS 4
#define CSA_OP_OUT_PROJ 5   /* Tq = T, N = g * d_g */
#define CSA_OP_INDEXER_MX 6 /* indexer_scores_topk_mxfp8 */

/* ---- (1) compression ------------------------------------------------ */

/*
 * CSA overlapped softmax-gated compression [§3.3 of the summary page: two
 * groups of KV entries and compression weights, a row softmax over 2m
 * elements, overlapping index ranges so that the rate is exactly 1/m].
 *   entry[b,s,ch] = sum_{j<m} sa_j kv_a[b,ms+j,ch] + sum_{j<m} sb_j kv_b[b,m(s-1)+j,ch]
 * with (sa, sb) = softmax over the 2m logits z_a[b,ms+j,.], z_b[b,m(s-1)+j,.]
 * taken per channel (z_cols == c) or per token (z_cols == 1); entry 0 has no
 * b group.  Each entry is then RMSNorm'd and rotated at position pos0 + m s.
 *   kv_a, kv_b, z_a, z_b: [B, T, c] ([B, T, z_cols] for the logits), `dtype`.
 *   entries (out): [B, floor(T/m), c].  Tail tokens (T mod m) make no entry.
 *   win_out (out, optional, may be NULL): [B, T, c] window rows
 *       RoPE_{pos0+j}(RMSNorm(kv_a[b,j])).
 *   ws: workspace of at least csa_workspace_bytes(CSA_OP_COMPRESS, ...) bytes
 *       (256: the status word), zeroed before first use; the streaming path
 *       records a copy wait that runs out there (CSA_DEV_TIMEOUT).
 * Errors: CSA_E_ARG for null/misaligned pointers or T < 0, m < 1;
 *         CSA_E_UNSUPPORTED for 2m > 256 or an unsupported c;
 *         CSA_E_WORKSPACE for a null or short ws (checked after the others,
 *         and only when there is work to launch).
 */
csa_status csa_compress(int32_t dtype, int64_t B, int64_t T, int32_t m, const csa_fmt* fmt,
                        const void* kv_a, const void* kv_b, const void* z_a, const void* z_b,
                        int32_t z_cols, int64_t pos0, void* entries, void* win_out, void* ws,
                        size_t ws_bytes, void* stream);

/*
 * HCA compression [§3.3 of the summary page: a larger rate m' with no
 * overlap, otherwise as CSA]:  entry[b,s] = sum_{j<m'} s_j kv[b,m's+j] with s
 * the per-channel softmax of z over the m' tokens of block s; then RMSNorm and
 * RoPE at pos0 + m' s.  kv, z: [B, T, c] / [B, T, z_cols]; entries:
 * [B, floor(T/m'), c]; win_out (optional): [B, T, c] = RoPE_{pos0+j}(RMSNorm(kv[b,j])).
 * ws as csa_compress.  Errors as csa_compress; m' up to 4096.
 */
csa_status hca_compress(int32_t dtype, int64_t B, int64_t T, int32_t m_prime, const csa_fmt* fmt,
                        const void* kv, const void* z, int32_t z_cols, int64_t pos0, void* entries,
                        void* win_out, void* ws, size_t ws_bytes, void* stream);

/* ---- (1b) streaming compression for decode ----------------------------- */

/*
 * Bytes of one sequence's stream state (a multiple of 256) for
 * csa_compress_append (overlap = 1, rate m) or hca_compress_append
 * (overlap = 0, rate m'): a 16-byte header holding the int64 count t of tokens
 * appended so far, then the tail buffer in the tensors' dtype -- the current
 * block's group-a rows and logits and, for CSA, the group-b rows and logits
 * of the current and the previous block.  Returns 0 for bad arguments.
 */
size_t csa_stream_state_bytes(int32_t dtype, int32_t m, int32_t overlap, int32_t c,
                              int32_t z_cols);

/*
 * Appends one token to each of B sequences' CSA compression state, as a decode
 * step produces them [§3.3 of the summary page: the entry of block s pools
 * the block's group-a rows and the previous block's group-b rows under a
 * per-channel softmax over the 2m logits; the page "DeepSeek-V4 梗概",
 * inference-infrastructure table, row "Tail buffer": the tokens of a block
 * that is not yet complete wait in a tail buffer].  For sequence b, with t the
 * token count stored in its state:
 *   - the token (kv_a[b], kv_b[b], z_a[b], z_b[b]) is stored in the tail
 *     buffer as slot t mod m of block s = t / m;
 *   - win_out[b] (optional) = RoPE_{pos0+t}(RMSNorm(kv_a[b])), its window row;
 *   - when t mod m == m - 1, entry s -- exactly what csa_compress produces for
 *     entry s of the whole sequence -- is written to entries[b, s];
 *   - t becomes t + 1.
 *   kv_a, kv_b: [B, c]; z_a, z_b: [B, z_cols] (dtype); state: B consecutive
 *   states of state_stride bytes each (>= csa_stream_state_bytes, a multiple
 *   of 16; zero-filled before a sequence's first token); entries: [B, n_cap,
 *   c] entry cache; win_out: [B, c] or NULL.  ws: >= 256 bytes (status word).
 * A state whose count is negative is skipped and an entry s >= n_cap is
 * dropped, both reported as CSA_DEV_STREAM.  Sequences are independent
 * (one CTA each): a sequence's results do not depend on the batch.
 * Errors: CSA_E_ARG (null or misaligned pointers, m < 1, bad z_cols or a
 * stride too small), CSA_E_UNSUPPORTED (2m > 256, c not in {64, ..., 1024} or
 * odd), CSA_E_WORKSPACE.
 */
csa_status csa_compress_append(int32_t dtype, int64_t B, int32_t m, const csa_fmt* fmt,
                               const void* kv_a, const void* kv_b, const void* z_a,
                               const void* z_b, int32_t z_cols, int64_t pos0, void* state,
                               size_t state_stride, void* entries, int64_t n_cap, void* win_out,
                               void* ws, size_t ws_bytes, void* stream);

/*
 * hca_compress_append: the same for an HCA layer [§3.3 of the summary page:
 * rate m', no overlap]: entry s pools the m' rows of block s.  kv, z: [B, c] /
 * [B, z_cols].  m' up to 4096.
 */
csa_status hca_compress_append(int32_t dtype, int64_t B, int32_t m_prime, const csa_fmt* fmt,
                               const void* kv, const void* z, int32_t z_cols, int64_t pos0,
                               void* state, size_t state_stride, void* entries, int64_t n_cap,
                               void* win_out, void* ws, size_t ws_bytes, void* stream);

/* ---- (1c) mixed BF16 / FP8 storage of compressed entries --------------- */

/*
 * Stores compressed entries in mixed precision [§3.3 of the summary page,
 * last paragraph: the KV entries keep their RoPE dims in BF16 and store the
 * rest in FP8].  Format taken (the page gives no block size or scale format):
 * the c - r non-RoPE dims as MX-FP8 (E4M3 codes, one UE8M0 scale per 32 dims,
 * 2^(floor(log2 amax) - 8), round to nearest even, saturate at 448), the r
 * RoPE dims rounded to bf16.  One record of csa_mixed_record_bytes(c, r)
 * bytes per entry (592 for c = 512, r = 64):
 *   bytes [0, c-r): E4M3 codes; [c-r, c+r): bf16 RoPE dims;
 *   [c+r, c+r+(c-r)/32): exponent + 127 per block; zeros to a multiple of 16.
 *   entries: [B, N, c] (dtype); records (out): [B, N, record bytes].
 * The attention calls read records in place of rows under CSA_F_MIXED.
 * Errors: CSA_E_ARG (null or misaligned pointers, negative sizes),
 * CSA_E_UNSUPPORTED ((c - r) not a multiple of 32, or c - r > 1024).
 */
size_t csa_mixed_record_bytes(int32_t c, int32_t rope_dims);
csa_status csa_store_mixed(int32_t dtype, int64_t B, int64_t N, const csa_fmt* fmt,
                           const void* entries, void* records, void* stream);

/* ---- (2) lightning indexer + top-k ----------------------------------- */

/*
 * Lightning-indexer scores and causal top-k [§3.3 of the summary page:
 * I[t,s] = sum_h w[t,h] ReLU(q_I[t,h] . K_I[s]); the top-k entries form the
 * candidate set].  For each (b, t) with position p = q_pos[b,t] (or t when
 * q_pos is NULL), the visible entries are s < min(N, floor((p+1)/m)); the
 * k_eff = min(k, visible) largest scores are selected, ties going to the lower
 * index, and emitted in ascending index order, padded with -1.
 *   q_I: [B, Tq, H_I, d_I] (dtype); w: [B, Tq, H_I] float32;
 *   k_I: [B, N, d_I] (dtype); q_pos: [B, Tq] int64 or NULL;
 *   idx_out: [B, Tq, k] int32; score_out: [B, Tq, k] float32 or NULL (the
 *   score of each selected index, -inf for padding).
 *   ws: workspace of at least csa_workspace_bytes(CSA_OP_INDEXER, ...) bytes,
 *   zero-filled once before its first use (status word at offset 0).
 * Arithmetic: bf16 products with float32 accumulation (exact for small
 * integer inputs); float32 throughout for CSA_F32.
 * Kernels: bf16 runs on the tensor cores, which need H_I = 64, d_I = 128,
 * B <= 65535 and ceil(Tq / 4) <= 65535; other bf16 shapes return
 * CSA_E_UNSUPPORTED.  float32 runs on CUDA cores for any H_I <= 64,
 * d_I <= 1024.  q_I and k_I must start on a 16-byte boundary (CSA_E_ARG).
 */
csa_status indexer_scores_topk(int32_t dtype, int64_t B, int64_t Tq, int32_t H_I, int32_t d_I,
                               const void* q_I, const float* w, const void* k_I, int64_t N,
                               const int64_t* q_pos, int32_t m, int32_t k, int32_t* idx_out,
                               float* score_out, void* ws, size_t ws_bytes, void* stream);

/*
 * indexer_scores_topk without a workspace.  The pages have no counterpart to
 * this call: it exists for callers that cannot allocate device memory where
 * they call the indexer (an engine plug-in whose host owns all device memory
 * through its own pool, or a decode loop that must not pay for cudaMalloc and
 * its implicit synchronisation).  Same arguments, checks and results as
 * indexer_scores_topk minus ws/ws_bytes.  Its scratch lives in a fixed 8 MiB
 * __device__ array inside libcsa.so that every GPU loading the library holds
 * until exit.  A call is accepted iff 256 (the status word) + the scratch of
 * the kernels it takes <= 8 MiB, else CSA_E_WORKSPACE: bf16 (tensor cores)
 * needs, when the entries span n_chunks > 1 chunks of 2048 (Tq >= 4) or 4096
 * (Tq < 4) entries, 4 * B * Tq * 4096 * n_chunks bytes for Tq < 4 and
 * n_chunks <= 16 (the raw score rows) and 8 * B * Tq * k * n_chunks bytes
 * otherwise (the chunks' candidates), and none for one chunk; float32 (CUDA
 * cores) needs 4 * B * Tq * N bytes.  For bf16 this equals
 * csa_workspace_bytes(CSA_OP_INDEXER, ...) <= 8 MiB.  The first call on each
 * device looks up the array's device address and caches it, so make that
 * first call before any stream capture.  All calls share the array and its
 * contents persist between calls: calls that overlap on the GPU race.
 * Kernel-side status is cleared per call and not reported: after a device-side
 * error (a bounded wait that ran out) the outputs are unspecified and nothing
 * tells the caller; use indexer_scores_topk with a workspace and
 * csa_check_status where that must be detected.  Nothing here calls
 * cudaMalloc, cudaFree or any allocating routine.
 */
csa_status indexer_scores_topk_noalloc(int32_t dtype, int64_t B, int64_t Tq, int32_t H_I,
                                       int32_t d_I, const void* q_I, const float* w,
                                       const void* k_I, int64_t N, const int64_t* q_pos,
                                       int32_t m, int32_t k, int32_t* idx_out, float* score_out,
                                       void* stream);

/* ---- (2b) low-precision indexer: MX-FP8 operands ------------------------ */

/*
 * The indexer's QK path in low precision [§3.3 of the summary page, last
 * paragraph, and §3.6: the indexer's query-key product runs in FP4 (the model
 * is trained for it) and keeps almost all of the full-precision selection].
 * Format taken: OCP Microscaling FP8 -- E4M3 elements with one power-of-two
 * scale per 32 consecutive elements of a 128-element row,
 * 2^(floor(log2 amax) - 8), elements rounded to nearest (ties to even) and
 * saturated at 448; the scale tensor is laid out for the block-scaled tensor
 * cores: per 128 rows of a batch element a 512-byte tile whose byte
 * 16 (r mod 32) + 4 (r div 32) + kb holds row r's block-kb exponent + 127
 * (0 for rows past the end).
 *   x: [B, rows, 128] (dtype CSA_BF16 or CSA_F32); codes (out): [B, rows,
 *   128] uint8; scales (out): [B, ceil(rows / 128), 512] uint8.
 * Used for the cached K_I (B sequences of N rows) and each step's q_I
 * (B Tq tokens of H_I = 64 rows: one tile per token).
 * Errors: CSA_E_ARG (null or misaligned pointers, negative sizes),
 * CSA_E_UNSUPPORTED (d != 128).
 */
csa_status indexer_mxfp8_quantize(int32_t dtype, int64_t B, int64_t rows, int32_t d,
                                  const void* x, void* codes, void* scales, void* stream);

/*
 * indexer_scores_topk on MX-FP8 operands (as indexer_mxfp8_quantize writes
 * them): I[t,s] = sum_h w[t,h] ReLU(sum_kb 2^(eq + ek) sum_{i in kb} cq_i ck_i)
 * with the E4M3 products and their sums in float32 on block-scaled tcgen05
 * MMAs; the causal top-k, tie rule, padding and outputs as indexer_scores_topk.
 *   q_codes: [B, Tq, 64, 128]; q_scales: [B, Tq, 512] (indexer_mxfp8_quantize
 *   of q_I as B Tq batch elements of 64 rows);
 *   k_codes: [B, N, 128]; k_scales: [B, ceil(N / 128), 512]; the others as
 *   indexer_scores_topk.  H_I must be 64 and d_I 128 (else CSA_E_UNSUPPORTED).
 *   ws: >= csa_workspace_bytes(CSA_OP_INDEXER_MX, CSA_BF16, B, Tq, 0, 0, N, k, 0).
 */
csa_status indexer_scores_topk_mxfp8(int64_t B, int64_t Tq, int32_t H_I, int32_t d_I,
                                     const void* q_codes, const void* q_scales, const float* w,
                                     const void* k_codes, const void* k_scales, int64_t N,
                                     const int64_t* q_pos, int32_t m, int32_t k, int32_t* idx_out,
                                     float* score_out, void* ws, size_t ws_bytes, void* stream);

/*
 * The same low-precision path with FP4, the precision the pages name for the
 * indexer ([§3.3 last paragraph and §3.6 of the summary page]).  Format taken:
 * OCP MX-FP4 -- E2M1 elements (magnitudes 0, 0.5, ..., 6) with one UE8M0
 * scale per 32 elements, 2^(floor(log2 amax) - 2), rounded to nearest (ties
 * to even) and saturated at 6, packed two to a byte (the even element in the
 * low nibble): codes [B, rows, 64] uint8; the scale tiles exactly as for
 * MX-FP8.  indexer_scores_topk_mxfp4 takes q_codes [B, Tq, 64, 64] and
 * k_codes [B, N, 64] (with their scale tiles) and runs block-scaled
 * kind::mxf4 MMAs (K = 64, two scales each); everything else as
 * indexer_scores_topk_mxfp8 (same workspace).
 */
csa_status indexer_mxfp4_quantize(int32_t dtype, int64_t B, int64_t rows, int32_t d,
                                  const void* x, void* codes, void* scales, void* stream);
csa_status indexer_scores_topk_mxfp4(int64_t B, int64_t Tq, int32_t H_I, int32_t d_I,
                                     const void* q_codes, const void* q_scales, const float* w,
                                     const void* k_codes, const void* k_scales, int64_t N,
                                     const int64_t* q_pos, int32_t m, int32_t k, int32_t* idx_out,
                                     float* score_out, void* ws, size_t ws_bytes, void* stream);

/* ---- (3) shared-KV MQA ------------------------------------------------ */

/*
 * Sparse MQA of a CSA layer [§3.3 of the summary page: MQA in which each
 * compressed entry is both key and value, over the top-k entries; RMSNorm on
 * the query; partial RoPE on query, entries and output, the output rotated
 * again at position -i; a sliding-window branch of n_win uncompressed rows.
 * The page "DeepSeek V4 完整技术报告" adds the learnable per-head sink logit].
 * For each (b, t, h), with p = q_pos[b,t] (or t):
 *   q^ = RoPE_p(RMSNorm(q[b,t,h]));
 *   keys = {entries[b, idx[b,t,i]] : idx >= 0} U {win[b, j - win_pos0[b]] :
 *           max(p - n_win + 1, win_pos0) <= j <= min(p, win_pos0 + Tw - 1)};
 *   out[b,t,h] = RoPE_{-p}( sum_key e^{l} key / (e^{sink[h]} + sum_key e^{l}) ),
 *   l = scale * q^ . key  (scale <= 0 means 1/sqrt(c); sink NULL means -inf).
 *   q: [B, Tq, H, c]; entries: [B, N, c]; idx: [B, Tq, k] int32 (-1 = none);
 *   win: [B, Tw, c]; win_pos0: [B] int64 or NULL (0); out: [B, Tq, H, c].
 * The bf16 tensor-core kernel requires the stored keys to be RMS-normalised
 * (as the compression calls produce them): it uses the static logit bound
 * scale*|q^|*sqrt(c) in place of a running maximum and flags CSA_DEV_RANGE
 * when a logit goes more than 60 (natural log) beyond it (the output is then
 * invalid).  An index outside [-1, N) is skipped and flagged CSA_DEV_BAD_INDEX.
 * With CSA_F_MIXED in fmt->flags, `entries` holds csa_store_mixed records
 * ([B, N, csa_mixed_record_bytes(c, r)] bytes; window rows stay dtype) and
 * the keys are the records' exact values (E4M3 x 2^e and bf16 both widen
 * exactly); the tensor cores then need rope_dims = 64.
 * Kernels: bf16 runs on the tensor cores, which need c = 512, H a multiple of
 * 64, rope_dims <= 64 and (sparse) k <= 1024; other bf16 shapes return
 * CSA_E_UNSUPPORTED unless fmt->flags has CSA_F_PORTABLE, which selects the
 * CUDA-core kernel (float32 always runs there; it keeps an exact running
 * maximum).
 */
csa_status sparse_mqa_attn(int32_t dtype, int64_t B, int64_t Tq, int32_t H, const csa_fmt* fmt,
                           const void* q, const int64_t* q_pos, const void* entries, int64_t N,
                           const int32_t* idx, int32_t k, const void* win, int64_t Tw,
                           const int64_t* win_pos0, int32_t n_win, const float* sink, float scale,
                           void* out, void* ws, size_t ws_bytes, void* stream);

/*
 * Dense MQA of an HCA layer [§3.3 of the summary page: HCA keeps dense
 * attention, otherwise as CSA]: as sparse_mqa_attn with the key set
 * {entries[b, s] : s < min(N, floor((p+1)/m_prime))} U window rows.
 */
csa_status dense_hca_attn(int32_t dtype, int64_t B, int64_t Tq, int32_t H, const csa_fmt* fmt,
                          const void* q, const int64_t* q_pos, const void* entries, int64_t N,
                          int32_t m_prime, const void* win, int64_t Tw, const int64_t* win_pos0,
                          int32_t n_win, const float* sink, float scale, void* out, void* ws,
                          size_t ws_bytes, void* stream);

/* ---- (4) grouped output projection ----------------------------------- */

/*
 * Grouped output projection of the attention output [§3.3 of the summary
 * page, CSA paragraph: c * n_h is large, so the heads' outputs are first
 * projected group by group to an intermediate dim d_g, then concatenated and
 * projected back to the model dim d].  The H heads split into g consecutive
 * groups of H/g heads (the reading taken: the pages give the map's shape,
 * not the grouping):
 *   v[t, j d_g + n] = sum_k o[t, j (H/g) c + k] w_group[j, n, k]   (o as [T, H c])
 *   y[t, n]         = sum_k v[t, k] w_out[n, k]
 *   o: [T, H, c] bf16; w_group: [g, d_g, (H/g) c] bf16; w_out: [d, g d_g] bf16;
 *   y (out): [T, d] bf16.  v lives in the workspace as bf16 (the products
 *   and sums of both GEMMs in float32; v and y rounded once to bf16).
 *   ws: >= csa_workspace_bytes(CSA_OP_OUT_PROJ, CSA_BF16, 1, T, 0, 0, g d_g, 0, 0)
 *   = 256 + 2 T g d_g bytes.
 * Tensor cores only: bf16 with H % g == 0, (H/g) c and g d_g multiples of 64,
 * d_g and d multiples of 32; anything else is CSA_E_UNSUPPORTED (float32
 * included).  Errors: CSA_E_ARG, CSA_E_UNSUPPORTED, CSA_E_WORKSPACE.
 */
csa_status grouped_output_projection(int32_t dtype, int64_t T, int32_t H, int32_t c, int32_t g,
                                     int32_t d_g, int32_t d, const void* o, const void* w_group,
                                     const void* w_out, void* y, void* ws, size_t ws_bytes,
                                     void* stream);

/* ---- workspace and status --------------------------------------------- */

/*
 * Bytes of workspace the op needs for these shapes (always >= 256: the
 * status word).  op: CSA_OP_*; unused arguments are ignored (k for the dense
 * op, H and c for the indexer).  Returns 0 for an unknown op.
 */
size_t csa_workspace_bytes(int32_t op, int32_t dtype, int64_t B, int64_t Tq, int32_t H, int32_t c,
                           int64_t N, int32_t k, int32_t n_win);

/*
 * Synchronises `stream`, reads the device status word at the start of `ws`
 * and clears it.  Returns CSA_OK, CSA_E_DEVICE (with *detail set to a
 * CSA_DEV_* code when detail != NULL), or CSA_E_CUDA.
 */
csa_status csa_check_status(void* ws, void* stream, uint32_t* detail);

/*
 * Failure-path self test: one CTA waits on an mbarrier that nothing
 * arrives on, with the same bounded wait every kernel here uses but a limit of
 * limit_ns nanoseconds (1e3 .. 1e10).  The wait runs out; the kernel
 * records CSA_DEV_TIMEOUT in the status word of `ws` (at least 256 bytes) and
 * returns, and the context stays usable.  csa_check_status() then reports
 * CSA_E_DEVICE with detail CSA_DEV_TIMEOUT.  Asynchronous on `stream`.
 * Errors: CSA_E_ARG (null ws, ws_bytes < 256, limit out of range),
 * CSA_E_CUDA.
 */
csa_status csa_selftest_wait(int64_t limit_ns, void* ws, size_t ws_bytes, void* stream);

/* Human-readable name of a status code (static storage). */
const char* csa_status_string(csa_status s);

/* Number of kernels this library has launched in this process so far (all
 * threads, all devices).  For launch accounting in benchmarks. */
unsigned long long csa_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* CSA_H_ */
