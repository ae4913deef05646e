/*
 * sws.h -- C ABI of libsws, the B200 (sm_100a) Sketch&Walk sparse-attention hot path.
 *
 * Source of the method: "Scout Before You Attend: Sketch-and-Walk Sparse Attention
 * for Efficient LLM Inference" (blog deep-dive of arXiv 2602.07397). Section numbers
 * below refer to that page.
 *
 * Conventions shared by every call
 *  - Pointers marked (device) are CUDA device pointers on the handle's device; (host)
 *    pointers are ordinary host memory. The caller owns every buffer. The library
 *    allocates device memory only in sws_create (the projection matrix) and never in
 *    a compute call.
 *  - Every device pointer must be 16-byte aligned; tensors are dense, row-major,
 *    with the layouts stated per call, except the per-head activations of the
 *    prefill calls, which take strides (see "Strided operands" below).
 *  - Compute calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *    stream) and return after the launches were queued. A call that fails its host-side
 *    validation returns a status and queues nothing. Launch failures return SWS_ERR_CUDA.
 *  - Device-side guards (bounded waits, index checks) never trap: they record a code in
 *    a per-device error word; sws_sync_check reads and clears it.
 *  - No C++ exception crosses this boundary.
 *
 * Notation: n tokens, B block size, b = ceil(n/B) blocks, d head dim, k sketch dim,
 * s walk power, hq query heads, hkv KV heads (query head h reads KV head h/(hq/hkv)),
 * density num/den, tau_i = ceil((i+1)*num/den) key blocks for query block i.
 *
 * Shape limits checked by every call: hkv >= 1, hkv divides hq, hq <= 4096
 * (SWS_ERR_INVALID_ARG otherwise); the prefill calls take b <= 8192 blocks
 * (SWS_ERR_UNSUPPORTED beyond).
 */
#ifndef SWS_H_
#define SWS_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SWS_OK = 0,
  SWS_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, bad size, inconsistent shapes */
  SWS_ERR_UNSUPPORTED = 2,  /* valid request outside what the kernels implement */
  SWS_ERR_WORKSPACE = 3,    /* workspace smaller than sws_workspace_size reports */
  SWS_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed */
  SWS_ERR_DEVICE_CHECK = 5  /* a device-side guard fired (see sws_sync_check) */
} sws_status;

typedef enum { SWS_BF16 = 0, SWS_FP32 = 1 } sws_dtype;

/* What (A_block)^s of §4 means: the matrix power (default), or the entrywise power
 * with rows renormalised to sum 1 (the alternative reading of "sparsity exponent"). */
typedef enum { SWS_WALK_MATRIX_POWER = 0, SWS_WALK_ELEMENTWISE = 1 } sws_walk_mode;

/* Operations whose workspace can be queried. */
typedef enum {
  SWS_OP_SKETCH = 0,
  SWS_OP_WALK_SELECT = 1,
  SWS_OP_PREFILL_ATTN = 2,
  SWS_OP_DECODE_ATTN = 3
} sws_op;

typedef struct {
  int32_t head_dim;    /* d: 64 or 128 */
  int32_t block_size;  /* B: 64 or 128 */
  int32_t sketch_dim;  /* k: 1..d (the page's default is 64; its ablation uses 16-32) */
  int32_t walk_power;  /* s: 1..64 (default 8, §7) */
  int32_t walk_mode;   /* sws_walk_mode */
  int32_t density_num; /* 0 < num <= den; 1/5 = the page's 20% density */
  int32_t density_den;
  int32_t select_group; /* query heads that share one selection: 0 or 1 = each head its own (the
                        * page's method); G > 1 = the G consecutive query heads of a GQA group
                        * share the top-tau of their summed walk rows (prefill) or of the
                        * log-sum-exp of their log-domain walk rows (decode). An extension the
                        * page does not define. Prefill needs G | hq; decode needs G = hq/hkv. */
  uint64_t seed;       /* seeds the random signs and columns of H_d */
} sws_config;

typedef struct sws_handle sws_handle;

/* ---------------------------------------------------------------- host-only --- */

const char* sws_status_string(sws_status s);

/* Checks a config against the limits above. Host only; never touches a GPU. */
sws_status sws_config_check(const sws_config* cfg);

/* Number of blocks b = ceil(n/B), or -1 for an invalid config or n < 1. */
int64_t sws_num_blocks(const sws_config* cfg, int64_t n);

/* Key blocks kept per head over all query blocks: sum over i < b of tau_i, or -1. */
int64_t sws_csr_nnz(const sws_config* cfg, int64_t n);

/* The Hadamard projection H_d of §3.2 (d x k, row-major doubles, host memory):
 * H_d = sqrt(d/k) * D * (H/sqrt(d)) * P, H the Sylvester Hadamard matrix, D random
 * signs, P k distinct columns. Signs and columns come from the splitmix64 stream
 * started at seed XOR 0x5357535F48414431: draws 0..d-1 give the signs (+1 when the
 * top bit is 0), the next d-1 draws a Fisher-Yates shuffle of [0, d) (for r = d-1
 * down to 1 swap r and draw mod (r+1)); P is the first k shuffled entries.
 * `hd` receives d*k doubles. */
sws_status sws_build_projection_host(const sws_config* cfg, double* hd);

/* Workspace bytes that `op` needs for the given sizes (batch is used by decode only). */
sws_status sws_workspace_size(const sws_config* cfg, sws_op op, int64_t n, int32_t hq, int32_t hkv,
                              int32_t batch, size_t* bytes);

/* --------------------------------------------------------------- handle --- */

/* Validates cfg and uploads H_d to the current CUDA device (the only allocation the
 * library makes). On failure *out is NULL. */
sws_status sws_create(const sws_config* cfg, sws_handle** out);
sws_status sws_destroy(sws_handle* h);

/* Device copy of H_d (d x k doubles, row-major), owned by the handle. */
const double* sws_projection_device(const sws_handle* h);

/* Number of kernels this library has queued in this process since it was loaded
 * (all devices, all threads). Host only; used to count launches in a timed region. */
uint64_t sws_launch_count(void);

/* Synchronises `stream`, then reads and clears the device error word.
 * Returns SWS_OK, SWS_ERR_DEVICE_CHECK (with *code = the recorded guard code), or SWS_ERR_CUDA. */
sws_status sws_sync_check(const sws_handle* h, void* stream, int32_t* code);

/* ---------------------------------------------------------------- prefill --- */
/* Strided operands. Q, K, V and O of the prefill calls are [heads, n, d] with the
 * d elements of each row contiguous; `x_strides` (host, two int64) gives the
 * element distance from one head to the next (x_strides[0]) and from one token to
 * the next (x_strides[1]), so row t of head h starts at x + h*x_strides[0] +
 * t*x_strides[1]. NULL means dense: {n*d, d}. A model's [n, heads, d] activations
 * are read in place with {d, heads*d}. Each stride must be at least d and a
 * multiple of 16 bytes (SWS_ERR_INVALID_ARG otherwise); every row addressed must
 * lie in the caller's allocation, and no two rows of O may overlap. */

/* Host only: SWS_OK when `strides` (NULL = dense) is valid for an operand of n
 * tokens of `dtype` under cfg (the check every prefill call makes), else
 * SWS_ERR_INVALID_ARG. */
sws_status sws_layout_check(const sws_config* cfg, sws_dtype dtype, int64_t n, const int64_t strides[2]);

/* sws_sketch. §3.1 block means (a partial last block divides by its row count),
 * §3.2 projection q~_i = q_bar_i H_d, k~_j = k_bar_j H_d and the sketched block scores
 * S[h,i,j] = q~_i(h) . k~_j(h/(hq/hkv)) / sqrt(k) for j <= i (causal block mask).
 *   q      (device) [hq, n, d]   dtype, strides q_strides (NULL: dense)
 *   k      (device) [hkv, n, d]  dtype, strides k_strides (NULL: dense)
 *   q_sk   (device) [hq, b, k]   double, written
 *   k_sk   (device) [hkv, b, k]  double, written
 *   scores (device) [hq, b, b]   double; entries j <= i written, j > i left untouched.
 *          May be NULL: then the scores are not formed here and the caller goes on
 *          with sws_walk_select_sketch, which forms them on chip from q_sk and k_sk.
 *   ws     (device) sws_workspace_size(SWS_OP_SKETCH) bytes, currently 0: the block
 *          means stay on chip (may be NULL while the size is 0)
 * Reads Q and K once: one fused pass forms the block means and projects them. */
sws_status sws_sketch(const sws_handle* h, const void* q, const void* k, sws_dtype dtype, int64_t n,
                      int32_t hq, int32_t hkv, const int64_t q_strides[2], const int64_t k_strides[2],
                      double* q_sk, double* k_sk, double* scores, void* ws, size_t ws_bytes, void* stream);

/* sws_walk_select. §4: A = row softmax of scores over j <= i (the sketched block
 * attention matrix), M = A^s, R = M on the first layer, else R = R_prev * M; then for
 * each query block i the tau_i largest R[i, j], j <= i (ties to the lower j), listed in
 * ascending order as CSR.
 *   scores     (device) [hq, b, b] double (lower triangle read)
 *   walk_state (device) [hq, b, b] double: R_prev in (ignored if first_layer), R out.
 *              Lower triangle written; entries above the diagonal are written as 0.
 *   row_ptr    (device) [hq, b+1] int32, written: offsets into the head's col_idx slice
 *   col_idx    (device) [hq, nnz] int32, written (nnz = sws_csr_nnz)
 *   ws         (device) sws_workspace_size(SWS_OP_WALK_SELECT) bytes
 * The walk runs in fp64: R spans hundreds of decades after a few layers. */
sws_status sws_walk_select(const sws_handle* h, const double* scores, int64_t n, int32_t hq, int first_layer,
                           double* walk_state, int32_t* row_ptr, int32_t* col_idx, void* ws, size_t ws_bytes,
                           void* stream);

/* sws_walk_select_sketch. The same walk and selection as sws_walk_select, from the
 * sketches instead of the score matrix: the sketched block scores of §3.2,
 * S[h,i,j] = q~_i(h) . k~_j(h/(hq/hkv)) / sqrt(k), are formed tile by tile on chip
 * (on the fp64 tensor path, the same products in the same order as sws_sketch
 * uses, so the same values) and go straight into the row softmax; the [hq, b, b]
 * score matrix never reaches device memory.
 *   q_sk (device) [hq, b, k] double, k_sk (device) [hkv, b, k] double: as
 *        sws_sketch wrote them
 *   walk_state, row_ptr, col_idx, ws: as sws_walk_select (same workspace size)
 * The row sums of the softmax are accumulated in another order than in
 * sws_walk_select, so the two calls agree to rounding (about 1e-15 relative). */
sws_status sws_walk_select_sketch(const sws_handle* h, const double* q_sk, const double* k_sk, int64_t n,
                                  int32_t hq, int32_t hkv, int first_layer, double* walk_state, int32_t* row_ptr,
                                  int32_t* col_idx, void* ws, size_t ws_bytes, void* stream);

/* sws_sparse_attn_prefill. §4/§5: exact softmax attention on the original Q, K, V
 * restricted to the selected key blocks; query token t attends to the tokens u of the
 * blocks listed for its block with u <= t. Online softmax, fp32 accumulation.
 *   q (device) [hq, n, d], k, v (device) [hkv, n, d], o (device) [hq, n, d]: all dtype,
 *     each with its strides (NULL: dense)
 *   row_ptr, col_idx: the CSR of sws_walk_select (each row ascending, within [0, i])
 * bf16 runs on the tensor cores (fp32 accumulate, output rounded to nearest);
 * fp32 runs in fp32 FMA. */
sws_status sws_sparse_attn_prefill(const sws_handle* h, const void* q, const void* k, const void* v,
                                   sws_dtype dtype, int64_t n, int32_t hq, int32_t hkv, const int64_t q_strides[2],
                                   const int64_t k_strides[2], const int64_t v_strides[2],
                                   const int64_t o_strides[2], const int32_t* row_ptr, const int32_t* col_idx,
                                   void* o, void* ws, size_t ws_bytes, void* stream);

/* sws_sparse_attn_prefill_varlen. The attention of sws_sparse_attn_prefill over
 * several sequences in one launch (the batching of prompts of different lengths that
 * §11.4 asks of serving): the sequences lie end to end along the token axis, sequence
 * s on rows cu_seqlens[s] .. cu_seqlens[s+1] - 1 of every head, and each is attended
 * with its own selection. The work of all sequences is one list, longest slabs first,
 * so short sequences fill the GPU together.
 *   q (device) [hq, N, d], k, v (device) [hkv, N, d], o (device) [hq, N, d]: bf16,
 *     N = cu_seqlens[nseq], each with its strides (NULL: dense)
 *   cu_seqlens (host) [nseq + 1] int64: 0 = cu_seqlens[0] < cu_seqlens[1] < ...,
 *     N < 2^31
 *   row_ptr, col_idx (host) arrays of nseq device pointers: sequence s's CSR, as
 *     sws_walk_select writes it for its n_s = cu_seqlens[s+1] - cu_seqlens[s] tokens
 *   ws (device, 16-byte aligned) sws_sparse_attn_prefill_varlen_ws_bytes bytes: the
 *     sequence table and the work list, copied there in stream order by this call
 * For finite inputs each sequence's rows of o equal, bit for bit, what
 * sws_sparse_attn_prefill writes for that sequence alone (the same tiles and the same
 * order of operations; keys past a sequence's end are masked in both). Rows of o
 * outside every sequence are not written. fp32 returns SWS_ERR_UNSUPPORTED.
 * The tables are copied from pageable host memory, so a stream that is being
 * captured into a CUDA graph rejects the call (SWS_ERR_CUDA). */
size_t sws_sparse_attn_prefill_varlen_ws_bytes(int32_t nseq, const int64_t* cu_seqlens);
sws_status sws_sparse_attn_prefill_varlen(const sws_handle* h, const void* q, const void* k, const void* v,
                                          sws_dtype dtype, int32_t nseq, const int64_t* cu_seqlens, int32_t hq,
                                          int32_t hkv, const int64_t q_strides[2], const int64_t k_strides[2],
                                          const int64_t v_strides[2], const int64_t o_strides[2],
                                          const int32_t* const* row_ptr, const int32_t* const* col_idx, void* o,
                                          void* ws, size_t ws_bytes, void* stream);

/* ----------------------------------------------------------------- decode --- */
/* §5: each decode step scores its single new query token against the cached key
 * blocks with the same sketch. The query is a block of one row; cached key blocks are
 * their means (the last, partial block by its count). A 1 x b row has no matrix
 * power, so over the layers of one step the walk is the entrywise product of the
 * per-layer rows raised to s, kept as logarithms:
 *   rho^l_j = rho^{l-1}_j + s * (z^l_j - logsumexp_j z^l),  z_j = q~ . k~_j / sqrt(k).
 * The new token is appended to the cache before it attends.
 *
 * Per-layer state (device, caller-owned):
 *   k_cache, v_cache [batch, hkv, max_len, d] bf16
 *   k_psum           [batch, hkv, d] double: sum of the keys of the last block
 *   k_sketch         [batch, hkv, max_blocks, k] double: sketched means of the cached blocks
 * with max_blocks = ceil(max_len/B). seq_lens (device, int32 [batch]) counts the tokens
 * of each sequence. */

/* Builds k_psum and k_sketch for caches that already hold seq_lens[i] tokens. */
sws_status sws_decode_init_cache(const sws_handle* h, const void* k_cache, int32_t batch, int32_t hkv,
                                 int64_t max_len, const int32_t* seq_lens, double* k_psum, double* k_sketch,
                                 void* stream);

/* Adds 1 to each of the batch entries of seq_lens (device). */
sws_status sws_decode_advance(const sws_handle* h, int32_t* seq_lens, int32_t batch, void* stream);

/* One layer of the decode-side sketch, walk and selection. seq_lens counts the tokens
 * INCLUDING this step's token, which is written at position seq_lens[i]-1.
 *   q_tok [batch, hq, d], k_tok / v_tok [batch, hkv, d] (device, bf16)
 *   walk_state [batch, hq, max_blocks] double: rho in (ignored if first_layer), out
 *   head_sel   [batch, hq, max_blocks] int32: each head's blocks, ascending; head_cnt [batch, hq]
 *   sel        [batch, hkv, max_blocks] int32: union over the GQA group, ascending
 *   sel_mask   [batch, hkv, max_blocks] uint8: bit r set = query head hkv_index*group + r chose it
 *   sel_cnt    [batch, hkv] int32
 * group = hq/hkv must be <= 8, and the selection's shared memory (about
 * max_blocks * (8 * group + 4) bytes: 5.6K blocks, 364K tokens at B = 64, for a group
 * of 4) must stay within 200 KB; SWS_ERR_UNSUPPORTED otherwise. */
sws_status sws_decode_step(const sws_handle* h, const void* q_tok, const void* k_tok, const void* v_tok,
                           int32_t batch, int32_t hq, int32_t hkv, int64_t max_len, const int32_t* seq_lens,
                           void* k_cache, void* v_cache, double* k_psum, double* k_sketch, int first_layer,
                           double* walk_state, int32_t* head_sel, int32_t* head_cnt, int32_t* sel,
                           uint8_t* sel_mask, int32_t* sel_cnt, void* stream);

/* The decode selection without the log-domain reduction: the row of the new token's
 * query block in the prefill recurrence of §4, R^l[i] = R^{l-1}[i] (A^l)^s, on the
 * sequence as it stands (prompt and decoded tokens). Over the layers of a step the row
 * is carried in walk_state (a probability row, not logarithms; do not mix with
 * sws_decode_step within a step) and advanced by s vector-matrix products with A^l,
 * the causal row softmax of q~_m . k~_j / sqrt(k) over every cached query and key block.
 * The selection then equals that of sws_walk_select for the last query block of a
 * prefill of the same tokens. It costs O(s b^2) per head and layer.
 *   q_psum   [batch, hq, d] double: sum of the queries of the last block
 *   q_sketch [batch, hq, max_blocks, k] double: q~ of every block (the prefill's q_sk)
 * Initialise both by calling sws_decode_init_cache on the prompt's queries, laid out
 * [batch, hq, max_len, d] with hkv = hq, next to the same call on the key cache. Other
 * arguments as sws_decode_step. Requires sketch_dim <= 32 and a multiple of 4, and the
 * per-CTA shared memory (a 4-byte triangle of max_blocks rows, one head's q~ and the
 * KV head's k~) to fit in 227 KB, which holds to about max_blocks = 260 at a GQA group
 * of 4 and d = 128; otherwise SWS_ERR_UNSUPPORTED. The block attention is held to a
 * relative 2^-21 (scores in fp32, each entry rounded to a 20-bit mantissa with the
 * fp64 exponent range); the products accumulate in fp64.
 * Matrix-power walks only (SWS_ERR_UNSUPPORTED for SWS_WALK_ELEMENTWISE). */
sws_status sws_decode_step_exact(const sws_handle* h, const void* q_tok, const void* k_tok, const void* v_tok,
                                 int32_t batch, int32_t hq, int32_t hkv, int64_t max_len, const int32_t* seq_lens,
                                 void* k_cache, void* v_cache, double* k_psum, double* k_sketch, double* q_psum,
                                 double* q_sketch, int first_layer, double* walk_state, int32_t* head_sel,
                                 int32_t* head_cnt, int32_t* sel, uint8_t* sel_mask, int32_t* sel_cnt, void* stream);

/* The exact decode walk above for contexts of any length (up to 2560 blocks: a
 * 163,840-token context at B = 64), with the rows of each layer's block attention
 * kept in device memory between steps. Row m of A^l (the causal row softmax of
 * q~_m . k~_j / sqrt(k), j <= m) no longer changes once block m is complete, so a
 * step writes only the newest block's row, and the s products read the stored
 * rows once per eight levels of s (a sweep from the newest block up to block 0).
 * The selection equals that of sws_decode_step_exact on the same state up to
 * rounding (the rows are formed by the same operations; the products add in
 * another order).
 *   rows (device) per layer: [batch, hq, E] uint32 with E = sws_decode_exact_rows_entries
 *        entries per (sequence, query head): row m holds columns 0..m, padded with
 *        zeros to a multiple of 4 entries, at entry offset 4(q+1)(2q+r) with
 *        q = m div 4, r = m mod 4; each entry is the high 32 bits of the fp64
 *        value rounded to nearest (sign, exponent, 20 mantissa bits).
 * Build them once, after sws_decode_init_cache has built the key and query
 * sketches of the prompt, with sws_decode_exact_rows_init; each call of
 * sws_decode_step_exact_rows then appends the token (as sws_decode_step_exact)
 * and rewrites the newest row before the products. Other arguments as
 * sws_decode_step_exact. Requires sketch_dim <= 32 and max_blocks <= 2560
 * (SWS_ERR_UNSUPPORTED otherwise). Memory: 4 E bytes per (sequence, query head,
 * layer), about 2 max_blocks^2 bytes (8.4 MB at 2049 blocks). */
int64_t sws_decode_exact_rows_entries(const sws_config* cfg, int64_t max_len);
sws_status sws_decode_exact_rows_init(const sws_handle* h, const double* q_sketch, const double* k_sketch,
                                      int32_t batch, int32_t hq, int32_t hkv, int64_t max_len,
                                      const int32_t* seq_lens, uint32_t* rows, void* stream);
sws_status sws_decode_step_exact_rows(const sws_handle* h, const void* q_tok, const void* k_tok, const void* v_tok,
                                      int32_t batch, int32_t hq, int32_t hkv, int64_t max_len,
                                      const int32_t* seq_lens, void* k_cache, void* v_cache, double* k_psum,
                                      double* k_sketch, double* q_psum, double* q_sketch, uint32_t* rows,
                                      int first_layer, double* walk_state, int32_t* head_sel, int32_t* head_cnt,
                                      int32_t* sel, uint8_t* sel_mask, int32_t* sel_cnt, void* stream);

/* sws_sparse_attn_decode: one query token per (sequence, head) over the tokens
 * (< seq_lens[i]) of the blocks its head selected. Each KV block of the group's union is
 * read once for all the group's heads (split over the union, then combined).
 *   q_tok [batch, hq, d] bf16; o [batch, hq, d] bf16 (device)
 *   ws    sws_workspace_size(SWS_OP_DECODE_ATTN) bytes
 * group = hq/hkv must be 1, 2, 4 or 8 (SWS_ERR_UNSUPPORTED otherwise). */
sws_status sws_sparse_attn_decode(const sws_handle* h, const void* q_tok, const void* k_cache,
                                  const void* v_cache, int32_t batch, int32_t hq, int32_t hkv, int64_t max_len,
                                  const int32_t* seq_lens, const int32_t* sel, const uint8_t* sel_mask,
                                  const int32_t* sel_cnt, void* o, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------ paged KV cache --- */
/* The same three decode calls over a paged cache: a pool of pages shared by all the
 * sequences of a batch, each page holding one key block (B tokens) of one sequence for
 * all of its KV heads, and a block table that maps each sequence's logical blocks to
 * pages. The pages have no counterpart in "Scout Before You Attend"; they let a
 * serving loop grow, share and free sequence storage block by block. Selection and
 * attention are the same as with the contiguous cache: the same pool content gives
 * the same result, bit for bit.
 *   k_pages, v_pages [num_pages, hkv, B, d] bf16 (device)
 *   block_table      [batch, max_blocks] int32 (device): the page of logical block j of
 *                    sequence i; entries past ceil(seq_lens[i] / B) are not read
 * A sequence holds at most max_blocks * B tokens (the max_len of the contiguous calls;
 * size k_sketch and walk_state with max_blocks, and query sws_workspace_size with
 * n = max_blocks * B). The step call writes the new token into its block's page, so
 * that page must be assigned before the call. A table entry outside [0, num_pages)
 * is not dereferenced: the block reads as empty (init, attention) or the token is not
 * appended, and guard code 6 is recorded for sws_sync_check. */
sws_status sws_decode_init_cache_paged(const sws_handle* h, const void* k_pages, int64_t num_pages,
                                       const int32_t* block_table, int64_t max_blocks, int32_t batch, int32_t hkv,
                                       const int32_t* seq_lens, double* k_psum, double* k_sketch, void* stream);
sws_status sws_decode_step_paged(const sws_handle* h, const void* q_tok, const void* k_tok, const void* v_tok,
                                 int32_t batch, int32_t hq, int32_t hkv, void* k_pages, void* v_pages,
                                 int64_t num_pages, const int32_t* block_table, int64_t max_blocks,
                                 const int32_t* seq_lens, double* k_psum, double* k_sketch, int first_layer,
                                 double* walk_state, int32_t* head_sel, int32_t* head_cnt, int32_t* sel,
                                 uint8_t* sel_mask, int32_t* sel_cnt, void* stream);
sws_status sws_sparse_attn_decode_paged(const sws_handle* h, const void* q_tok, const void* k_pages,
                                        const void* v_pages, int64_t num_pages, const int32_t* block_table,
                                        int64_t max_blocks, int32_t batch, int32_t hq, int32_t hkv,
                                        const int32_t* seq_lens, const int32_t* sel, const uint8_t* sel_mask,
                                        const int32_t* sel_cnt, void* o, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------- no-allocation variant --- */
/* The paper has no counterpart to this call; it serves callers that cannot allocate
 * device memory on the decode path (a plug-in whose host framework owns every device
 * allocation, a serving loop that may not pay an allocation's latency and implicit
 * synchronisation per token, a fixed memory budget decided up front).
 *
 * Same computation, arguments and layouts as sws_sparse_attn_decode, without the
 * workspace: the split-KV partial results go to one scratch array of
 * SWS_NOALLOC_SCRATCH_BYTES built into the library. The CUDA runtime places that array
 * on every device the library is loaded on, and it stays there until the process exits.
 *  - The call allocates nothing (no cudaMalloc, no cudaFree, nothing through a framework).
 *  - sws_create looks up the array's device address (cudaGetSymbolAddress) with the
 *    handle's device current and keeps it in the handle, so this call does no set-up of
 *    its own. The address belongs to the CUDA context the handle was created in: after
 *    that context is torn down (cudaDeviceReset), create a new handle.
 *  - The handle's device must be the current device.
 *  - Every call shares the one array and finds the previous call's contents in it (each
 *    call overwrites all it reads). Calls whose kernels overlap on the GPU race on it:
 *    issue them on one stream, or order them.
 *  - Returns SWS_ERR_WORKSPACE, and queues nothing, when batch * hq * splits * (d + 2) * 4
 *    bytes of partials (what sws_workspace_size(SWS_OP_DECODE_ATTN) reports) would exceed
 *    SWS_NOALLOC_SCRATCH_BYTES; the workspace form has no such limit. */
#define SWS_NOALLOC_SCRATCH_BYTES (32u << 20)
sws_status sws_sparse_attn_decode_noalloc(const sws_handle* h, const void* q_tok, const void* k_cache,
                                          const void* v_cache, int32_t batch, int32_t hq, int32_t hkv,
                                          int64_t max_len, const int32_t* seq_lens, const int32_t* sel,
                                          const uint8_t* sel_mask, const int32_t* sel_cnt, void* o, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SWS_H_ */
