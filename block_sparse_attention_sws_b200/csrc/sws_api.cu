// libsws C ABI: argument validation, the projection builder, handle lifetime
// and the launch sequence of every entry point. No allocation happens here
// except in sws_create.
#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <vector>

#include "sws_common.cuh"

using namespace sws;

namespace sws {
static std::atomic<uint64_t> g_launches{0};
void note_launches(int count) { g_launches.fetch_add(static_cast<uint64_t>(count), std::memory_order_relaxed); }
}  // namespace sws

namespace {

bool aligned16(const void* p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool log_enabled() {
  static int on = -1;
  if (on < 0) {
    const char* e = std::getenv("SWS_LOG");
    on = (e && e[0] == '1') ? 1 : 0;
  }
  return on == 1;
}

sws_status cuda_status(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return SWS_OK;
  if (log_enabled()) std::fprintf(stderr, "[sws] %s: %s\n", what, cudaGetErrorString(e));
  return SWS_ERR_CUDA;
}

bool pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

// splitmix64 (Steele, Lea and Flood, OOPSLA 2014): state advance + output mix.
uint64_t splitmix_next(uint64_t& state) {
  state += 0x9E3779B97F4A7C15ull;
  uint64_t z = state;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

constexpr uint64_t kProjectionTag = 0x5357535F48414431ull;

int popcount32(uint32_t x) {
  int c = 0;
  while (x) {
    x &= x - 1;
    ++c;
  }
  return c;
}

sws_status check_heads(int32_t hq, int32_t hkv) {
  if (hq < 1 || hkv < 1 || hq % hkv != 0 || hq > 4096) return SWS_ERR_INVALID_ARG;
  return SWS_OK;
}

constexpr int64_t kMaxPrefillBlocks = 8192;  // top-tau counters and row staging limit

}  // namespace

namespace {

sws_status decode_init_cache(const sws_handle* h, const void* k_cache, const KvLayout& kv, int32_t batch,
                             const int32_t* seq_lens, double* k_psum, double* k_sketch, void* stream) {
  if (!aligned16(k_cache) || !aligned16(seq_lens) || !aligned16(k_psum) || !aligned16(k_sketch))
    return SWS_ERR_INVALID_ARG;
  return cuda_status(launch_decode_init_cache(h, static_cast<const __nv_bfloat16*>(k_cache), kv, batch, seq_lens,
                                              k_psum, k_sketch, static_cast<cudaStream_t>(stream)),
                     "decode init cache");
}

sws_status decode_step(const sws_handle* h, const void* q_tok, const void* k_tok, const void* v_tok, int32_t batch,
                       int32_t hq, const KvLayout& kv, const int32_t* seq_lens, void* k_cache, void* v_cache,
                       double* k_psum, double* k_sketch, int first_layer, double* walk_state, int32_t* head_sel,
                       int32_t* head_cnt, int32_t* sel, uint8_t* sel_mask, int32_t* sel_cnt, void* stream) {
  if (!h || batch < 1 || check_heads(hq, kv.hkv) != SWS_OK) return SWS_ERR_INVALID_ARG;
  if (hq / kv.hkv > 8) return SWS_ERR_UNSUPPORTED;
  if (h->cfg.select_group > 1 && h->cfg.select_group != hq / kv.hkv) return SWS_ERR_INVALID_ARG;
  const void* ptrs[] = {q_tok, k_tok, v_tok, seq_lens, k_cache, v_cache, k_psum, k_sketch,
                        walk_state, head_sel, head_cnt, sel, sel_mask, sel_cnt};
  for (const void* p : ptrs)
    if (!aligned16(p)) return SWS_ERR_INVALID_ARG;
  if (decode_select_smem_bytes(h->cfg, kv.max_blocks, hq / kv.hkv) > (200u << 10)) return SWS_ERR_UNSUPPORTED;
  return cuda_status(
      launch_decode_select(h, static_cast<const __nv_bfloat16*>(q_tok), static_cast<const __nv_bfloat16*>(k_tok),
                           static_cast<const __nv_bfloat16*>(v_tok), batch, hq, kv, seq_lens,
                           static_cast<__nv_bfloat16*>(k_cache), static_cast<__nv_bfloat16*>(v_cache), k_psum,
                           k_sketch, first_layer, walk_state, head_sel, head_cnt, sel, sel_mask, sel_cnt,
                           static_cast<cudaStream_t>(stream)),
      "decode step");
}

sws_status sparse_attn_decode(const sws_handle* h, const void* q_tok, const void* k_cache, const void* v_cache,
                              int32_t batch, int32_t hq, const KvLayout& kv, const int32_t* seq_lens,
                              const int32_t* sel, const uint8_t* sel_mask, const int32_t* sel_cnt, void* o, void* ws,
                              size_t ws_bytes, void* stream) {
  if (!h || batch < 1 || check_heads(hq, kv.hkv) != SWS_OK) return SWS_ERR_INVALID_ARG;
  const int32_t group = hq / kv.hkv;
  if (group != 1 && group != 2 && group != 4 && group != 8) return SWS_ERR_UNSUPPORTED;
  const void* ptrs[] = {q_tok, k_cache, v_cache, seq_lens, sel, sel_mask, sel_cnt, o, ws};
  for (const void* p : ptrs)
    if (!aligned16(p)) return SWS_ERR_INVALID_ARG;
  size_t need = 0;
  if (sws_workspace_size(&h->cfg, SWS_OP_DECODE_ATTN, kv.max_len, hq, kv.hkv, batch, &need) != SWS_OK)
    return SWS_ERR_INVALID_ARG;
  if (ws_bytes < need) return SWS_ERR_WORKSPACE;
  const int32_t splits = decode_num_splits(h->cfg, kv.max_len, group);
  return cuda_status(launch_decode_attn(h, static_cast<const __nv_bfloat16*>(q_tok),
                                        static_cast<const __nv_bfloat16*>(k_cache),
                                        static_cast<const __nv_bfloat16*>(v_cache), batch, hq, kv, seq_lens, sel,
                                        sel_mask, sel_cnt, static_cast<__nv_bfloat16*>(o), static_cast<float*>(ws),
                                        splits, static_cast<cudaStream_t>(stream)),
                     "decode attention");
}

// a paged pool: [num_pages, hkv, B, d] pages and a [batch, max_blocks] table
bool paged_args_ok(int32_t hkv, int64_t num_pages, const int32_t* block_table, int64_t max_blocks) {
  return hkv >= 1 && num_pages >= 1 && num_pages <= INT32_MAX && max_blocks >= 1 && max_blocks <= (INT32_MAX / 4096) &&
         aligned16(block_table);
}

}  // namespace

extern "C" {

const char* sws_status_string(sws_status s) {
  switch (s) {
    case SWS_OK: return "ok";
    case SWS_ERR_INVALID_ARG: return "invalid argument";
    case SWS_ERR_UNSUPPORTED: return "unsupported configuration";
    case SWS_ERR_WORKSPACE: return "workspace too small";
    case SWS_ERR_CUDA: return "CUDA error";
    case SWS_ERR_DEVICE_CHECK: return "device-side check failed";
  }
  return "unknown status";
}

sws_status sws_config_check(const sws_config* c) {
  if (!c) return SWS_ERR_INVALID_ARG;
  if (c->select_group < 0 || c->select_group > 8) return SWS_ERR_INVALID_ARG;
  if (c->head_dim != 64 && c->head_dim != 128) return SWS_ERR_UNSUPPORTED;
  if (c->block_size != 64 && c->block_size != 128) return SWS_ERR_UNSUPPORTED;
  if (c->sketch_dim < 1 || c->sketch_dim > c->head_dim) return SWS_ERR_INVALID_ARG;
  if (c->walk_power < 1 || c->walk_power > 64) return SWS_ERR_INVALID_ARG;
  if (c->walk_mode != SWS_WALK_MATRIX_POWER && c->walk_mode != SWS_WALK_ELEMENTWISE) return SWS_ERR_INVALID_ARG;
  if (c->density_num < 1 || c->density_den < 1 || c->density_num > c->density_den) return SWS_ERR_INVALID_ARG;
  if (!pow2(c->head_dim)) return SWS_ERR_UNSUPPORTED;
  return SWS_OK;
}

int64_t sws_num_blocks(const sws_config* c, int64_t n) {
  if (sws_config_check(c) != SWS_OK || n < 1) return -1;
  return ceil_div64(n, c->block_size);
}

int64_t sws_csr_nnz(const sws_config* c, int64_t n) {
  const int64_t b = sws_num_blocks(c, n);
  if (b < 0) return -1;
  int64_t nnz = 0;
  for (int64_t i = 0; i < b; ++i) nnz += tau_of_row(i, c->density_num, c->density_den);
  return nnz;
}

// Signs and the column permutation of the projection (its first k entries
// are the sampled columns), from the splitmix64 stream of the seed.
static void projection_draws(const sws_config* c, std::vector<int>& sign, std::vector<int>& perm) {
  const int d = c->head_dim;
  uint64_t state = c->seed ^ kProjectionTag;
  std::vector<uint64_t> draws(2 * d - 1);
  for (auto& x : draws) x = splitmix_next(state);
  sign.assign(d, 1);
  perm.resize(d);
  for (int r = 0; r < d; ++r) sign[r] = (draws[r] >> 63) ? -1 : 1;
  for (int r = 0; r < d; ++r) perm[r] = r;
  int next = d;
  for (int r = d - 1; r >= 1; --r) {
    const int j = static_cast<int>(draws[next++] % static_cast<uint64_t>(r + 1));
    std::swap(perm[r], perm[j]);
  }
}

// 1/sqrt(k), formed as sqrt(d/k)/sqrt(d) like every entry of H_d
static double projection_scale(const sws_config* c) {
  const int d = c->head_dim, k = c->sketch_dim;
  return std::sqrt(static_cast<double>(d) / k) / std::sqrt(static_cast<double>(d));
}

sws_status sws_build_projection_host(const sws_config* c, double* hd) {
  sws_status s = sws_config_check(c);
  if (s != SWS_OK) return s;
  if (!hd) return SWS_ERR_INVALID_ARG;
  const int d = c->head_dim, k = c->sketch_dim;
  std::vector<int> sign, perm;
  projection_draws(c, sign, perm);
  // H_d[r][c] = sqrt(d/k) * sign[r] * (-1)^popcount(r & perm[c]) / sqrt(d) = sign * (+-1) / sqrt(k)
  const double scale = projection_scale(c);
  for (int r = 0; r < d; ++r)
    for (int cc = 0; cc < k; ++cc) {
      const int par = popcount32(static_cast<uint32_t>(r & perm[cc])) & 1;
      hd[r * k + cc] = scale * sign[r] * (par ? -1.0 : 1.0);
    }
  return SWS_OK;
}

sws_status sws_workspace_size(const sws_config* c, sws_op op, int64_t n, int32_t hq, int32_t hkv, int32_t batch,
                              size_t* bytes) {
  sws_status s = sws_config_check(c);
  if (s != SWS_OK) return s;
  if (!bytes || n < 1 || check_heads(hq, hkv) != SWS_OK) return SWS_ERR_INVALID_ARG;
  const int64_t b = ceil_div64(n, c->block_size);
  switch (op) {
    case SWS_OP_SKETCH:
      *bytes = sketch_workspace_bytes(*c, n, hq, hkv);
      return SWS_OK;
    case SWS_OP_PREFILL_ATTN:
      *bytes = 0;
      return SWS_OK;
    case SWS_OP_WALK_SELECT:
      // up to four b x b fp64 matrices per head live at once (power by squaring)
      *bytes = 4 * static_cast<size_t>(hq) * b * b * sizeof(double);
      return SWS_OK;
    case SWS_OP_DECODE_ATTN: {
      if (batch < 1) return SWS_ERR_INVALID_ARG;
      const int32_t splits = decode_num_splits(*c, n, hq / hkv);
      *bytes = static_cast<size_t>(batch) * hq * splits * (c->head_dim + 2) * sizeof(float);
      return SWS_OK;
    }
  }
  return SWS_ERR_INVALID_ARG;
}

sws_status sws_create(const sws_config* c, sws_handle** out) {
  if (!out) return SWS_ERR_INVALID_ARG;
  *out = nullptr;
  sws_status s = sws_config_check(c);
  if (s != SWS_OK) return s;
  const int d = c->head_dim, k = c->sketch_dim;
  std::vector<double> hd(static_cast<size_t>(d) * k), hdt(static_cast<size_t>(d) * k);
  sws_build_projection_host(c, hd.data());
  for (int r = 0; r < d; ++r)
    for (int cc = 0; cc < k; ++cc) hdt[(size_t)cc * d + r] = hd[(size_t)r * k + cc];
  auto* h = new sws_handle();
  h->cfg = *c;
  cudaError_t e = cudaGetDevice(&h->device);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, h->device);
  std::vector<int> sign_i, perm;
  projection_draws(c, sign_i, perm);
  std::vector<double> sign(sign_i.begin(), sign_i.end());
  std::vector<int32_t> col(perm.begin(), perm.begin() + k);
  h->scale = projection_scale(c);
  void* mem = nullptr;
  const size_t hd_bytes = hd.size() * sizeof(double);
  const size_t sign_bytes = static_cast<size_t>(d) * sizeof(double);
  const size_t col_bytes = (static_cast<size_t>(k) * sizeof(int32_t) + 15) & ~size_t(15);
  if (e == cudaSuccess) e = cudaMalloc(&mem, 2 * hd_bytes + sign_bytes + col_bytes + 256);
  if (e != cudaSuccess) {
    delete h;
    return cuda_status(e, "sws_create");
  }
  h->hd = static_cast<double*>(mem);
  h->hdt = h->hd + hd.size();
  h->sign = h->hdt + hd.size();
  h->col = reinterpret_cast<int32_t*>(h->sign + d);
  h->err = reinterpret_cast<int32_t*>(reinterpret_cast<uint8_t*>(mem) + 2 * hd_bytes + sign_bytes + col_bytes);
  e = cudaMemcpy(h->hd, hd.data(), hd_bytes, cudaMemcpyHostToDevice);
  if (e == cudaSuccess) e = cudaMemcpy(h->hdt, hdt.data(), hd_bytes, cudaMemcpyHostToDevice);
  if (e == cudaSuccess) e = cudaMemcpy(h->sign, sign.data(), sign_bytes, cudaMemcpyHostToDevice);
  if (e == cudaSuccess) e = cudaMemcpy(h->col, col.data(), k * sizeof(int32_t), cudaMemcpyHostToDevice);
  if (e == cudaSuccess) e = cudaMemset(h->err, 0, sizeof(int32_t));
  if (e == cudaSuccess) e = noalloc_scratch_address(&h->noalloc_scratch);
  if (e != cudaSuccess) {
    cudaFree(mem);
    delete h;
    return cuda_status(e, "sws_create upload");
  }
  *out = h;
  return SWS_OK;
}

sws_status sws_destroy(sws_handle* h) {
  if (!h) return SWS_ERR_INVALID_ARG;
  cudaError_t e = cudaFree(h->hd);
  delete h;
  return cuda_status(e, "sws_destroy");
}

const double* sws_projection_device(const sws_handle* h) { return h ? h->hd : nullptr; }

uint64_t sws_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

sws_status sws_sync_check(const sws_handle* h, void* stream, int32_t* code) {
  if (!h) return SWS_ERR_INVALID_ARG;
  auto st = static_cast<cudaStream_t>(stream);
  int32_t v = 0;
  cudaError_t e = cudaStreamSynchronize(st);
  if (e == cudaSuccess) e = cudaMemcpy(&v, h->err, sizeof(v), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess && v != 0) e = cudaMemset(h->err, 0, sizeof(int32_t));
  if (code) *code = v;
  if (e != cudaSuccess) return cuda_status(e, "sws_sync_check");
  return v ? SWS_ERR_DEVICE_CHECK : SWS_OK;
}

extern "C++" {
namespace {

// The element strides of a [heads, n, d] operand (NULL: dense). Rows keep their
// d elements contiguous; both strides must move by whole rows (at least d) and by
// multiples of 16 bytes, so that every row starts 16-byte aligned.
bool head_tok(const int64_t* strides, int64_t n, int32_t d, size_t elem, HeadTok* out) {
  if (!strides) {
    *out = HeadTok{n * d, d};
    return true;
  }
  const int64_t hs = strides[0], ts = strides[1];
  if (hs < d || ts < d) return false;
  if ((hs * static_cast<int64_t>(elem)) % 16 != 0 || (ts * static_cast<int64_t>(elem)) % 16 != 0) return false;
  *out = HeadTok{hs, ts};
  return true;
}

}  // namespace
}  // extern "C++"

sws_status sws_layout_check(const sws_config* cfg, sws_dtype dtype, int64_t n, const int64_t strides[2]) {
  if (sws_config_check(cfg) != SWS_OK || n < 1 || (dtype != SWS_BF16 && dtype != SWS_FP32))
    return SWS_ERR_INVALID_ARG;
  HeadTok ht{};
  return head_tok(strides, n, cfg->head_dim, dtype == SWS_BF16 ? 2 : 4, &ht) ? SWS_OK : SWS_ERR_INVALID_ARG;
}

sws_status sws_sketch(const sws_handle* h, const void* q, const void* k, sws_dtype dtype, int64_t n, int32_t hq,
                      int32_t hkv, const int64_t q_strides[2], const int64_t k_strides[2], double* q_sk,
                      double* k_sk, double* scores, void* ws, size_t ws_bytes, void* stream) {
  if (!h || n < 1 || check_heads(hq, hkv) != SWS_OK) return SWS_ERR_INVALID_ARG;
  if (dtype != SWS_BF16 && dtype != SWS_FP32) return SWS_ERR_INVALID_ARG;
  const size_t elem = dtype == SWS_BF16 ? 2 : 4;
  HeadTok qs{}, ks{};
  if (!head_tok(q_strides, n, h->cfg.head_dim, elem, &qs) || !head_tok(k_strides, n, h->cfg.head_dim, elem, &ks))
    return SWS_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(q_sk) || !aligned16(k_sk) || (scores && !aligned16(scores)) ||
      (ws && !aligned16(ws)))
    return SWS_ERR_INVALID_ARG;
  const int64_t b = ceil_div64(n, h->cfg.block_size);
  if (b > kMaxPrefillBlocks) return SWS_ERR_UNSUPPORTED;
  if (ws_bytes < sketch_workspace_bytes(h->cfg, n, hq, hkv)) return SWS_ERR_WORKSPACE;
  auto st = static_cast<cudaStream_t>(stream);
  sws_status s = cuda_status(
      launch_sketch_pool_project(h, q, k, dtype, n, hq, hkv, qs, ks, q_sk, k_sk, st), "sketch pool+project");
  if (s != SWS_OK || !scores) return s;
  return cuda_status(launch_sketch_scores(h, q_sk, k_sk, b, hq, hkv, scores, st), "sketch scores");
}

extern "C++" {
namespace {

// The walk and the selection after the block attention matrix: M = A^s by
// binary powering (matrix power) or M = A (the entrywise power is folded into
// the softmax's temperature), R = M or R_prev M, then top-tau. `softmax`
// writes A into the buffer it is given.
template <typename Softmax>
sws_status walk_chain(const sws_handle* h, int64_t b, int32_t hq, int first_layer, double* walk_state,
                      int32_t* row_ptr, int32_t* col_idx, void* ws, cudaStream_t st, Softmax softmax) {
  const size_t mat = static_cast<size_t>(hq) * b * b;
  double* buf[4] = {static_cast<double*>(ws), static_cast<double*>(ws) + mat, static_cast<double*>(ws) + 2 * mat,
                    static_cast<double*>(ws) + 3 * mat};
  bool busy[4] = {false, false, false, false};
  // At most four products are live at once (base, result, the new product,
  // and R_prev * M after the loop), so take() always finds a free buffer; a
  // failure would be a bug in the schedule below and is reported, not used.
  auto take = [&]() -> int {
    for (int q = 0; q < 4; ++q)
      if (!busy[q]) {
        busy[q] = true;
        return q;
      }
    return -1;
  };
  const int a = take();
  sws_status s = cuda_status(softmax(buf[a]), "block softmax");
  if (s != SWS_OK) return s;
  int m_idx = a;  // holds M = A^s when done
  if (h->cfg.walk_mode == SWS_WALK_MATRIX_POWER && h->cfg.walk_power > 1) {
    // binary powering: result = prod of base^(2^t) over the set bits of s
    int base = a, result = -1;
    int e = h->cfg.walk_power;
    while (true) {
      if (e & 1) {
        if (result < 0) {
          result = base;
        } else {
          const int dst = take();
          if (dst < 0) return SWS_ERR_UNSUPPORTED;
          s = cuda_status(launch_tri_gemm(buf[result], buf[base], buf[dst], b, hq, st), "walk power");
          if (s != SWS_OK) return s;
          if (result != base) busy[result] = false;
          result = dst;
        }
      }
      e >>= 1;
      if (!e) break;
      const int dst = take();
      if (dst < 0) return SWS_ERR_UNSUPPORTED;
      s = cuda_status(launch_tri_gemm(buf[base], buf[base], buf[dst], b, hq, st), "walk square");
      if (s != SWS_OK) return s;
      if (base != result) busy[base] = false;
      base = dst;
    }
    if (base != result) busy[base] = false;
    m_idx = result;
  }
  const double* Rnew = buf[m_idx];
  if (!first_layer) {
    const int dst = take();
    if (dst < 0) return SWS_ERR_UNSUPPORTED;
    s = cuda_status(launch_tri_gemm(walk_state, buf[m_idx], buf[dst], b, hq, st), "walk update");
    if (s != SWS_OK) return s;
    Rnew = buf[dst];
  }
  return cuda_status(launch_select(h, Rnew, b, hq, walk_state, row_ptr, col_idx, st), "top-tau select");
}

// Checks shared by both walk-select entry points; b on success.
sws_status walk_args(const sws_handle* h, int64_t n, int32_t hq, int32_t hkv, const double* walk_state,
                     const int32_t* row_ptr, const int32_t* col_idx, const void* ws, size_t ws_bytes, int64_t* b) {
  if (!h || n < 1 || check_heads(hq, hkv) != SWS_OK) return SWS_ERR_INVALID_ARG;
  if (h->cfg.select_group > 1 && hq % h->cfg.select_group != 0) return SWS_ERR_INVALID_ARG;
  if (!aligned16(walk_state) || !aligned16(row_ptr) || !aligned16(col_idx) || !aligned16(ws))
    return SWS_ERR_INVALID_ARG;
  *b = ceil_div64(n, h->cfg.block_size);
  if (*b > kMaxPrefillBlocks) return SWS_ERR_UNSUPPORTED;
  size_t need = 0;
  if (sws_workspace_size(&h->cfg, SWS_OP_WALK_SELECT, n, hq, hkv, 1, &need) != SWS_OK) return SWS_ERR_INVALID_ARG;
  if (ws_bytes < need) return SWS_ERR_WORKSPACE;
  return SWS_OK;
}

}  // namespace
}  // extern "C++"

sws_status sws_walk_select(const sws_handle* h, const double* scores, int64_t n, int32_t hq, int first_layer,
                           double* walk_state, int32_t* row_ptr, int32_t* col_idx, void* ws, size_t ws_bytes,
                           void* stream) {
  int64_t b = 0;
  const sws_status v = walk_args(h, n, hq, 1, walk_state, row_ptr, col_idx, ws, ws_bytes, &b);
  if (v != SWS_OK) return v;
  if (!aligned16(scores)) return SWS_ERR_INVALID_ARG;
  auto st = static_cast<cudaStream_t>(stream);
  return walk_chain(h, b, hq, first_layer, walk_state, row_ptr, col_idx, ws, st,
                    [&](double* A) { return launch_block_softmax(h, scores, b, hq, A, st); });
}

sws_status sws_walk_select_sketch(const sws_handle* h, const double* q_sk, const double* k_sk, int64_t n, int32_t hq,
                                  int32_t hkv, int first_layer, double* walk_state, int32_t* row_ptr,
                                  int32_t* col_idx, void* ws, size_t ws_bytes, void* stream) {
  int64_t b = 0;
  const sws_status v = walk_args(h, n, hq, hkv, walk_state, row_ptr, col_idx, ws, ws_bytes, &b);
  if (v != SWS_OK) return v;
  if (!aligned16(q_sk) || !aligned16(k_sk)) return SWS_ERR_INVALID_ARG;
  auto st = static_cast<cudaStream_t>(stream);
  return walk_chain(h, b, hq, first_layer, walk_state, row_ptr, col_idx, ws, st,
                    [&](double* A) { return launch_sketch_softmax(h, q_sk, k_sk, b, hq, hkv, A, st); });
}

sws_status sws_sparse_attn_prefill(const sws_handle* h, const void* q, const void* k, const void* v,
                                   sws_dtype dtype, int64_t n, int32_t hq, int32_t hkv, const int64_t q_strides[2],
                                   const int64_t k_strides[2], const int64_t v_strides[2],
                                   const int64_t o_strides[2], const int32_t* row_ptr, const int32_t* col_idx,
                                   void* o, void* ws, size_t ws_bytes, void* stream) {
  (void)ws;
  (void)ws_bytes;
  if (!h || n < 1 || check_heads(hq, hkv) != SWS_OK) return SWS_ERR_INVALID_ARG;
  if (dtype != SWS_BF16 && dtype != SWS_FP32) return SWS_ERR_INVALID_ARG;
  const size_t elem = dtype == SWS_BF16 ? 2 : 4;
  const int32_t d = h->cfg.head_dim;
  PrefillLayout lay{};
  if (!head_tok(q_strides, n, d, elem, &lay.q) || !head_tok(k_strides, n, d, elem, &lay.k) ||
      !head_tok(v_strides, n, d, elem, &lay.v) || !head_tok(o_strides, n, d, elem, &lay.o))
    return SWS_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(row_ptr) || !aligned16(col_idx))
    return SWS_ERR_INVALID_ARG;
  if (ceil_div64(n, h->cfg.block_size) > kMaxPrefillBlocks) return SWS_ERR_UNSUPPORTED;
  auto st = static_cast<cudaStream_t>(stream);
  if (dtype == SWS_BF16)
    return cuda_status(launch_attn_prefill_tc(h, q, k, v, n, hq, hkv, lay, row_ptr, col_idx, o, st),
                       "prefill attention (tensor cores)");
  return cuda_status(launch_attn_prefill_simt(h, q, k, v, dtype, n, hq, hkv, lay, row_ptr, col_idx, o, st),
                     "prefill attention (fp32)");
}

size_t sws_sparse_attn_prefill_varlen_ws_bytes(int32_t nseq, const int64_t* cu_seqlens) {
  if (nseq < 1 || !cu_seqlens) return 0;
  for (int32_t s = 0; s < nseq; ++s)
    if (cu_seqlens[s + 1] <= cu_seqlens[s]) return 0;
  return attn_prefill_varlen_ws_bytes(nseq, cu_seqlens);
}

sws_status sws_sparse_attn_prefill_varlen(const sws_handle* h, const void* q, const void* k, const void* v,
                                          sws_dtype dtype, int32_t nseq, const int64_t* cu_seqlens, int32_t hq,
                                          int32_t hkv, const int64_t q_strides[2], const int64_t k_strides[2],
                                          const int64_t v_strides[2], const int64_t o_strides[2],
                                          const int32_t* const* row_ptr, const int32_t* const* col_idx, void* o,
                                          void* ws, size_t ws_bytes, void* stream) {
  if (!h || nseq < 1 || !cu_seqlens || !row_ptr || !col_idx || check_heads(hq, hkv) != SWS_OK)
    return SWS_ERR_INVALID_ARG;
  if (dtype != SWS_BF16) return dtype == SWS_FP32 ? SWS_ERR_UNSUPPORTED : SWS_ERR_INVALID_ARG;
  if (cu_seqlens[0] != 0) return SWS_ERR_INVALID_ARG;
  for (int32_t s = 0; s < nseq; ++s) {
    if (cu_seqlens[s + 1] <= cu_seqlens[s]) return SWS_ERR_INVALID_ARG;
    if (!aligned16(row_ptr[s]) || !aligned16(col_idx[s])) return SWS_ERR_INVALID_ARG;
    if (ceil_div64(cu_seqlens[s + 1] - cu_seqlens[s], h->cfg.block_size) > kMaxPrefillBlocks)
      return SWS_ERR_UNSUPPORTED;
  }
  const int64_t ntot = cu_seqlens[nseq];
  if (ntot > INT32_MAX - 2 * 128) return SWS_ERR_UNSUPPORTED;  // token coordinates of the tensor maps
  const int32_t d = h->cfg.head_dim;
  PrefillLayout lay{};
  if (!head_tok(q_strides, ntot, d, 2, &lay.q) || !head_tok(k_strides, ntot, d, 2, &lay.k) ||
      !head_tok(v_strides, ntot, d, 2, &lay.v) || !head_tok(o_strides, ntot, d, 2, &lay.o))
    return SWS_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(ws)) return SWS_ERR_INVALID_ARG;
  if (ws_bytes < attn_prefill_varlen_ws_bytes(nseq, cu_seqlens)) return SWS_ERR_WORKSPACE;
  return cuda_status(launch_attn_prefill_tc_varlen(h, q, k, v, hq, hkv, lay, nseq, cu_seqlens, row_ptr, col_idx, o,
                                                   ws, static_cast<cudaStream_t>(stream)),
                     "prefill attention (packed sequences)");
}

sws_status sws_decode_init_cache(const sws_handle* h, const void* k_cache, int32_t batch, int32_t hkv,
                                 int64_t max_len, const int32_t* seq_lens, double* k_psum, double* k_sketch,
                                 void* stream) {
  if (!h || batch < 1 || hkv < 1 || max_len < 1) return SWS_ERR_INVALID_ARG;
  return decode_init_cache(h, k_cache, contiguous_kv(h->cfg, hkv, max_len), batch, seq_lens, k_psum, k_sketch,
                           stream);
}

sws_status sws_decode_init_cache_paged(const sws_handle* h, const void* k_pages, int64_t num_pages,
                                       const int32_t* block_table, int64_t max_blocks, int32_t batch, int32_t hkv,
                                       const int32_t* seq_lens, double* k_psum, double* k_sketch, void* stream) {
  if (!h || batch < 1 || !paged_args_ok(hkv, num_pages, block_table, max_blocks)) return SWS_ERR_INVALID_ARG;
  return decode_init_cache(h, k_pages, paged_kv(h->cfg, hkv, block_table, max_blocks, num_pages), batch, seq_lens,
                           k_psum, k_sketch, stream);
}

sws_status sws_decode_advance(const sws_handle* h, int32_t* seq_lens, int32_t batch, void* stream) {
  if (!h || batch < 1 || !aligned16(seq_lens)) return SWS_ERR_INVALID_ARG;
  return cuda_status(launch_decode_advance(seq_lens, batch, static_cast<cudaStream_t>(stream)), "decode advance");
}

sws_status sws_decode_step(const sws_handle* h, const void* q_tok, const void* k_tok, const void* v_tok,
                           int32_t batch, int32_t hq, int32_t hkv, int64_t max_len, const int32_t* seq_lens,
                           void* k_cache, void* v_cache, double* k_psum, double* k_sketch, int first_layer,
                           double* walk_state, int32_t* head_sel, int32_t* head_cnt, int32_t* sel,
                           uint8_t* sel_mask, int32_t* sel_cnt, void* stream) {
  if (!h || max_len < 1 || hkv < 1) return SWS_ERR_INVALID_ARG;
  return decode_step(h, q_tok, k_tok, v_tok, batch, hq, contiguous_kv(h->cfg, hkv, max_len), seq_lens, k_cache,
                     v_cache, k_psum, k_sketch, first_layer, walk_state, head_sel, head_cnt, sel, sel_mask, sel_cnt,
                     stream);
}

sws_status sws_decode_step_exact(const sws_handle* h, const void* q_tok, const void* k_tok, const void* v_tok,
                                 int32_t batch, int32_t hq, int32_t hkv, int64_t max_len, const int32_t* seq_lens,
                                 void* k_cache, void* v_cache, double* k_psum, double* k_sketch, double* q_psum,
                                 double* q_sketch, int first_layer, double* walk_state, int32_t* head_sel,
                                 int32_t* head_cnt, int32_t* sel, uint8_t* sel_mask, int32_t* sel_cnt, void* stream) {
  if (!h || batch < 1 || max_len < 1 || check_heads(hq, hkv) != SWS_OK) return SWS_ERR_INVALID_ARG;
  if (h->cfg.select_group > 1 && h->cfg.select_group != hq / hkv) return SWS_ERR_INVALID_ARG;
  if (h->cfg.walk_mode != SWS_WALK_MATRIX_POWER) return SWS_ERR_UNSUPPORTED;
  const void* ptrs[] = {q_tok, k_tok, v_tok, seq_lens, k_cache, v_cache, k_psum, k_sketch, q_psum, q_sketch,
                        walk_state, head_sel, head_cnt, sel, sel_mask, sel_cnt};
  for (const void* p : ptrs)
    if (!aligned16(p)) return SWS_ERR_INVALID_ARG;
  if (!decode_exact_supported(h->cfg, ceil_div64(max_len, h->cfg.block_size), hq / hkv)) return SWS_ERR_UNSUPPORTED;
  return cuda_status(
      launch_decode_exact(h, static_cast<const __nv_bfloat16*>(q_tok), static_cast<const __nv_bfloat16*>(k_tok),
                          static_cast<const __nv_bfloat16*>(v_tok), batch, hq, hkv, max_len, seq_lens,
                          static_cast<__nv_bfloat16*>(k_cache), static_cast<__nv_bfloat16*>(v_cache), k_psum, k_sketch,
                          q_psum, q_sketch, first_layer, walk_state, head_sel, head_cnt, sel, sel_mask, sel_cnt,
                          static_cast<cudaStream_t>(stream)),
      "decode step (exact walk)");
}

int64_t sws_decode_exact_rows_entries(const sws_config* cfg, int64_t max_len) {
  if (sws_config_check(cfg) != SWS_OK || max_len < 1) return -1;
  return exact_rows_entries(ceil_div64(max_len, cfg->block_size));
}

sws_status sws_decode_exact_rows_init(const sws_handle* h, const double* q_sketch, const double* k_sketch,
                                      int32_t batch, int32_t hq, int32_t hkv, int64_t max_len,
                                      const int32_t* seq_lens, uint32_t* rows, void* stream) {
  if (!h || batch < 1 || max_len < 1 || check_heads(hq, hkv) != SWS_OK) return SWS_ERR_INVALID_ARG;
  const void* ptrs[] = {q_sketch, k_sketch, seq_lens, rows};
  for (const void* p : ptrs)
    if (!aligned16(p)) return SWS_ERR_INVALID_ARG;
  if (!exact_wide_supported(h->cfg, ceil_div64(max_len, h->cfg.block_size), hq / hkv)) return SWS_ERR_UNSUPPORTED;
  return cuda_status(launch_exact_rows_init(h, q_sketch, k_sketch, batch, hq, hkv, max_len, seq_lens, rows,
                                            static_cast<cudaStream_t>(stream)),
                     "exact walk rows");
}

sws_status sws_decode_step_exact_rows(const sws_handle* h, const void* q_tok, const void* k_tok, const void* v_tok,
                                      int32_t batch, int32_t hq, int32_t hkv, int64_t max_len,
                                      const int32_t* seq_lens, void* k_cache, void* v_cache, double* k_psum,
                                      double* k_sketch, double* q_psum, double* q_sketch, uint32_t* rows,
                                      int first_layer, double* walk_state, int32_t* head_sel, int32_t* head_cnt,
                                      int32_t* sel, uint8_t* sel_mask, int32_t* sel_cnt, void* stream) {
  if (!h || batch < 1 || max_len < 1 || check_heads(hq, hkv) != SWS_OK) return SWS_ERR_INVALID_ARG;
  if (h->cfg.select_group > 1 && h->cfg.select_group != hq / hkv) return SWS_ERR_INVALID_ARG;
  if (h->cfg.walk_mode != SWS_WALK_MATRIX_POWER) return SWS_ERR_UNSUPPORTED;
  const void* ptrs[] = {q_tok, k_tok, v_tok, seq_lens, k_cache, v_cache, k_psum, k_sketch, q_psum, q_sketch,
                        rows, walk_state, head_sel, head_cnt, sel, sel_mask, sel_cnt};
  for (const void* p : ptrs)
    if (!aligned16(p)) return SWS_ERR_INVALID_ARG;
  if (!exact_wide_supported(h->cfg, ceil_div64(max_len, h->cfg.block_size), hq / hkv)) return SWS_ERR_UNSUPPORTED;
  return cuda_status(
      launch_decode_exact_wide(h, static_cast<const __nv_bfloat16*>(q_tok), static_cast<const __nv_bfloat16*>(k_tok),
                               static_cast<const __nv_bfloat16*>(v_tok), batch, hq, hkv, max_len, seq_lens,
                               static_cast<__nv_bfloat16*>(k_cache), static_cast<__nv_bfloat16*>(v_cache), k_psum,
                               k_sketch, q_psum, q_sketch, rows, first_layer, walk_state, head_sel, head_cnt, sel,
                               sel_mask, sel_cnt, static_cast<cudaStream_t>(stream)),
      "decode step (exact walk, stored rows)");
}

sws_status sws_decode_step_paged(const sws_handle* h, const void* q_tok, const void* k_tok, const void* v_tok,
                                 int32_t batch, int32_t hq, int32_t hkv, void* k_pages, void* v_pages,
                                 int64_t num_pages, const int32_t* block_table, int64_t max_blocks,
                                 const int32_t* seq_lens, double* k_psum, double* k_sketch, int first_layer,
                                 double* walk_state, int32_t* head_sel, int32_t* head_cnt, int32_t* sel,
                                 uint8_t* sel_mask, int32_t* sel_cnt, void* stream) {
  if (!h || !paged_args_ok(hkv, num_pages, block_table, max_blocks)) return SWS_ERR_INVALID_ARG;
  return decode_step(h, q_tok, k_tok, v_tok, batch, hq, paged_kv(h->cfg, hkv, block_table, max_blocks, num_pages),
                     seq_lens, k_pages, v_pages, k_psum, k_sketch, first_layer, walk_state, head_sel, head_cnt, sel,
                     sel_mask, sel_cnt, stream);
}

sws_status sws_sparse_attn_decode(const sws_handle* h, const void* q_tok, const void* k_cache, const void* v_cache,
                                  int32_t batch, int32_t hq, int32_t hkv, int64_t max_len, const int32_t* seq_lens,
                                  const int32_t* sel, const uint8_t* sel_mask, const int32_t* sel_cnt, void* o,
                                  void* ws, size_t ws_bytes, void* stream) {
  if (!h || max_len < 1 || hkv < 1) return SWS_ERR_INVALID_ARG;
  return sparse_attn_decode(h, q_tok, k_cache, v_cache, batch, hq, contiguous_kv(h->cfg, hkv, max_len), seq_lens,
                            sel, sel_mask, sel_cnt, o, ws, ws_bytes, stream);
}

sws_status sws_sparse_attn_decode_paged(const sws_handle* h, const void* q_tok, const void* k_pages,
                                        const void* v_pages, int64_t num_pages, const int32_t* block_table,
                                        int64_t max_blocks, int32_t batch, int32_t hq, int32_t hkv,
                                        const int32_t* seq_lens, const int32_t* sel, const uint8_t* sel_mask,
                                        const int32_t* sel_cnt, void* o, void* ws, size_t ws_bytes, void* stream) {
  if (!h || !paged_args_ok(hkv, num_pages, block_table, max_blocks)) return SWS_ERR_INVALID_ARG;
  return sparse_attn_decode(h, q_tok, k_pages, v_pages, batch, hq,
                            paged_kv(h->cfg, hkv, block_table, max_blocks, num_pages), seq_lens, sel, sel_mask,
                            sel_cnt, o, ws, ws_bytes, stream);
}

}  // extern "C"
