// Internal declarations shared by the libsws translation units.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "sws.h"

struct sws_handle {
  sws_config cfg;
  int device;
  int num_sms;
  double* hd;    // [d, k] row-major
  double* hdt;   // [k, d] row-major (transpose, for contiguous per-output reads)
  double* sign;  // [d] the random signs D of H_d (+1 / -1)
  int32_t* col;  // [k] the sampled Hadamard columns P of H_d
  double scale;  // 1/sqrt(k): H_d[r][c] = scale * sign[r] * (-1)^popcount(r & col[c])
  int32_t* err;  // device error word (guard code of the first failure, 0 = none)
  void* noalloc_scratch;  // device address of the built-in decode scratch in this handle's context
};

namespace sws {

// Codes recorded in the device error word.
enum Guard : int32_t {
  GUARD_NONE = 0,
  GUARD_MBAR_TIMEOUT = 1,  // a bounded mbarrier wait ran out
  GUARD_BAD_CSR = 2,       // a CSR entry outside [0, i] or a non-ascending row
  GUARD_BAD_SELECT = 3,    // top-tau bookkeeping inconsistent
  GUARD_BAD_LEN = 4,       // a sequence length outside [1, max_len]
  GUARD_TMEM = 5,          // tensor memory allocation failed
  GUARD_BAD_PAGE = 6       // a block table entry outside [0, num_pages)
};

__device__ __forceinline__ void record_error(int32_t* err, int32_t code) {
  if (err) atomicCAS(err, 0, code);
}

// ---- programmatic dependent launch ------------------------------------------
// Every kernel of the library is launched with programmatic stream
// serialisation (launch_k below), so that it can be scheduled while the
// previous kernel of the stream drains. Each kernel therefore calls
// grid_dependency_wait() before its first access to global memory (the wait
// returns once the previous grid has completed and its writes are visible; it
// is a no-op when there is no such grid), and allow_dependents() once it has
// started, which lets the next kernel be scheduled when every CTA of this one
// has issued it or exited.
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void allow_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ---- mbarrier / bulk-copy helpers (sm_90+ PTX, used on sm_100a) -------------

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// try_wait that suspends at most `hint_ns` nanoseconds before reporting "not yet".
__device__ __forceinline__ bool mbar_try_wait_hint(uint64_t* bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Waits are bounded in wall time (the global nanosecond timer), never by an
// iteration count: a wait that has not completed after kWaitNs gives up.
constexpr uint64_t kWaitNs = 1000000000ull;  // 1 s
constexpr uint32_t kSuspendNs = 20000;       // at most 20 us per try

// Bounded wait. Returns false, after recording the guard, on timeout.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int32_t* err) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  while (true) {
    if (mbar_try_wait_hint(bar, parity, kSuspendNs)) return true;
    if (global_ns() - t0 > kWaitNs) break;
  }
  record_error(err, GUARD_MBAR_TIMEOUT);
  return false;
}

// 1-D bulk copy global -> shared, completion counted on `bar` (bytes % 16 == 0,
// both addresses 16-byte aligned).
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// ---- conversions ------------------------------------------------------------

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// ---- integer helpers shared by host and device -------------------------------

__host__ __device__ __forceinline__ int64_t ceil_div64(int64_t a, int64_t b) { return (a + b - 1) / b; }

// tau_i = ceil((i+1) * num / den): key blocks kept for query block i.
__host__ __device__ __forceinline__ int32_t tau_of_row(int64_t i, int32_t num, int32_t den) {
  return static_cast<int32_t>(((i + 1) * static_cast<int64_t>(num) + den - 1) / den);
}

// ---- launchers (defined in the kernel translation units) ----------------------

// Counts queued kernels (sws_launch_count); every launcher calls it per launch.
void note_launches(int count);

// Launches kern<<<grid, block, smem, st>>>(args...) with programmatic stream
// serialisation allowed (see grid_dependency_wait).
template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t lc = {};
  lc.gridDim = grid;
  lc.blockDim = block;
  lc.dynamicSmemBytes = smem;
  lc.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = attr;
  lc.numAttrs = 1;
  return cudaLaunchKernelEx(&lc, kern, std::forward<Args>(args)...);
}

// Element strides of a [heads, tokens, d] operand whose rows of d elements are
// contiguous: row t of head h starts at base + h * head + t * tok.
struct HeadTok {
  int64_t head, tok;
};
// The four operands of prefill attention.
struct PrefillLayout {
  HeadTok q, k, v, o;
};

size_t sketch_workspace_bytes(const sws_config& c, int64_t n, int32_t hq, int32_t hkv);
cudaError_t launch_sketch_pool_project(const sws_handle* h, const void* q, const void* k, sws_dtype dt, int64_t n,
                                       int32_t hq, int32_t hkv, HeadTok qs, HeadTok ks, double* q_sk, double* k_sk,
                                       cudaStream_t st);
cudaError_t launch_sketch_scores(const sws_handle* h, const double* q_sk, const double* k_sk, int64_t b, int32_t hq,
                                 int32_t hkv, double* scores, cudaStream_t st);

cudaError_t launch_block_softmax(const sws_handle* h, const double* scores, int64_t b, int32_t hq, double* A,
                                 cudaStream_t st);
cudaError_t launch_sketch_softmax(const sws_handle* h, const double* q_sk, const double* k_sk, int64_t b, int32_t hq,
                                  int32_t hkv, double* A, cudaStream_t st);
cudaError_t launch_tri_gemm(const double* A, const double* Bm, double* C, int64_t b, int32_t hq, cudaStream_t st);
cudaError_t launch_select(const sws_handle* h, const double* R, int64_t b, int32_t hq, double* walk_state,
                          int32_t* row_ptr, int32_t* col_idx, cudaStream_t st);

cudaError_t launch_attn_prefill_simt(const sws_handle* h, const void* q, const void* k, const void* v, sws_dtype dt,
                                     int64_t n, int32_t hq, int32_t hkv, const PrefillLayout& lay,
                                     const int32_t* row_ptr, const int32_t* col_idx, void* o, cudaStream_t st);

size_t attn_prefill_varlen_ws_bytes(int32_t nseq, const int64_t* cu_seqlens);
cudaError_t launch_attn_prefill_tc_varlen(const sws_handle* h, const void* q, const void* k, const void* v,
                                          int32_t hq, int32_t hkv, const PrefillLayout& lay, int32_t nseq,
                                          const int64_t* cu_seqlens, const int32_t* const* row_ptr,
                                          const int32_t* const* col_idx, void* o, void* ws, cudaStream_t st);
cudaError_t launch_attn_prefill_tc(const sws_handle* h, const void* q, const void* k, const void* v, int64_t n,
                                   int32_t hq, int32_t hkv, const PrefillLayout& lay, const int32_t* row_ptr,
                                   const int32_t* col_idx, void* o, cudaStream_t st);

// Where the cached keys (or values) of one (sequence, KV head) live.
//  contiguous (block_table null): [batch, hkv, max_len, D]; token t of the unit
//    (sequence i, KV head g) is row (i * hkv + g) * max_len + t.
//  paged: a pool of pages [num_pages, hkv, B, D], one page per key block of a
//    sequence (all its KV heads); block_table[i * max_blocks + j] is the page of
//    logical block j of sequence i, so token t is row t % B of page
//    block_table[i * max_blocks + t / B]. max_len = max_blocks * B.
struct KvLayout {
  const int32_t* block_table;
  int64_t max_len;     // tokens a sequence can hold
  int64_t max_blocks;  // ceil(max_len / B)
  int64_t num_pages;
  int32_t hkv, B, D;
};

inline KvLayout contiguous_kv(const sws_config& c, int32_t hkv, int64_t max_len) {
  return KvLayout{nullptr, max_len, ceil_div64(max_len, c.block_size), 0, hkv, c.block_size, c.head_dim};
}
inline KvLayout paged_kv(const sws_config& c, int32_t hkv, const int32_t* block_table, int64_t max_blocks,
                         int64_t num_pages) {
  return KvLayout{block_table, max_blocks * c.block_size, max_blocks, num_pages, hkv, c.block_size, c.head_dim};
}

// Element offset of the first row of logical block j of (sequence bi, KV
// head g), or -1 when the block table points outside the pool.
__device__ __forceinline__ int64_t kv_block_offset(const KvLayout& L, int64_t bi, int64_t g, int64_t j) {
  if (!L.block_table) return ((bi * L.hkv + g) * L.max_len + j * L.B) * L.D;
  const int64_t p = L.block_table[bi * L.max_blocks + j];
  if (p < 0 || p >= L.num_pages) return -1;
  return ((p * L.hkv + g) * L.B) * L.D;
}

cudaError_t launch_decode_init_cache(const sws_handle* h, const __nv_bfloat16* k_cache, const KvLayout& kv,
                                     int32_t batch, const int32_t* seq_lens, double* k_psum, double* k_sketch,
                                     cudaStream_t st);
cudaError_t launch_decode_advance(int32_t* seq_lens, int32_t batch, cudaStream_t st);
cudaError_t launch_decode_select(const sws_handle* h, const __nv_bfloat16* q_tok, const __nv_bfloat16* k_tok,
                                 const __nv_bfloat16* v_tok, int32_t batch, int32_t hq, const KvLayout& kv,
                                 const int32_t* seq_lens, __nv_bfloat16* k_cache, __nv_bfloat16* v_cache,
                                 double* k_psum, double* k_sketch, int first_layer, double* walk_state,
                                 int32_t* head_sel, int32_t* head_cnt, int32_t* sel, uint8_t* sel_mask,
                                 int32_t* sel_cnt, cudaStream_t st);
cudaError_t launch_decode_exact(const sws_handle* h, const __nv_bfloat16* q_tok, const __nv_bfloat16* k_tok,
                                const __nv_bfloat16* v_tok, int32_t batch, int32_t hq, int32_t hkv, int64_t max_len,
                                const int32_t* seq_lens, __nv_bfloat16* k_cache, __nv_bfloat16* v_cache,
                                double* k_psum, double* k_sketch, double* q_psum, double* q_sketch, int first_layer,
                                double* walk_state, int32_t* head_sel, int32_t* head_cnt, int32_t* sel,
                                uint8_t* sel_mask, int32_t* sel_cnt, cudaStream_t st);
int64_t exact_rows_entries(int64_t max_blocks);
bool exact_wide_supported(const sws_config& c, int64_t max_blocks, int32_t group);
cudaError_t launch_exact_rows_init(const sws_handle* h, const double* q_sketch, const double* k_sketch, int32_t batch,
                                   int32_t hq, int32_t hkv, int64_t max_len, const int32_t* seq_lens, uint32_t* rows,
                                   cudaStream_t st);
cudaError_t launch_decode_exact_wide(const sws_handle* h, const __nv_bfloat16* q_tok, const __nv_bfloat16* k_tok,
                                     const __nv_bfloat16* v_tok, int32_t batch, int32_t hq, int32_t hkv,
                                     int64_t max_len, const int32_t* seq_lens, __nv_bfloat16* k_cache,
                                     __nv_bfloat16* v_cache, double* k_psum, double* k_sketch, double* q_psum,
                                     double* q_sketch, uint32_t* rows, int first_layer, double* walk_state,
                                     int32_t* head_sel, int32_t* head_cnt, int32_t* sel, uint8_t* sel_mask,
                                     int32_t* sel_cnt, cudaStream_t st);
size_t decode_exact_smem_bytes(const sws_config& cfg, int64_t max_blocks, int32_t group);
bool decode_exact_supported(const sws_config& cfg, int64_t max_blocks, int32_t group);
int32_t decode_num_splits(const sws_config& cfg, int64_t max_len, int32_t group);
cudaError_t noalloc_scratch_address(void** out);
size_t decode_select_smem_bytes(const sws_config& cfg, int64_t max_blocks, int32_t group);
cudaError_t launch_decode_attn(const sws_handle* h, const __nv_bfloat16* q_tok, const __nv_bfloat16* k_cache,
                               const __nv_bfloat16* v_cache, int32_t batch, int32_t hq, const KvLayout& kv,
                               const int32_t* seq_lens, const int32_t* sel, const uint8_t* sel_mask,
                               const int32_t* sel_cnt, __nv_bfloat16* o, float* partial, int32_t splits,
                               cudaStream_t st);

}  // namespace sws
