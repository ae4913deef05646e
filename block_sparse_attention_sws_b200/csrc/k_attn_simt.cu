// sw_sparse_attn_prefill in plain fp32 FMA (fp32 inputs).
//
// "Scout Before You Attend" §4/§5: exact softmax attention over the original
// Q, K, V restricted to the key blocks selected for each query block. Token t
// of query block i attends to the tokens u of the listed blocks with u <= t.
//
// One CTA per (query head, query block), two threads per query row (each owns
// half of the head dimension). Each selected key block is staged in shared
// memory; the block's scores are computed, then the running max / sum and the
// output accumulators are rescaled once per block (online softmax).
#include <algorithm>

#include "sws_common.cuh"

namespace sws {
namespace {

template <typename T, int D, int B>
__global__ void __launch_bounds__(2 * B) attn_simt_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                          const T* __restrict__ v, int64_t n, int32_t group,
                                                          PrefillLayout lay, const int32_t* __restrict__ row_ptr,
                                                          const int32_t* __restrict__ col_idx, int64_t nnz,
                                                          T* __restrict__ o, float qscale, int32_t* err) {
  grid_dependency_wait();
  allow_dependents();
  constexpr int HD = D / 2;
  constexpr int VE = 16 / sizeof(T);
  extern __shared__ __align__(16) uint8_t smem[];
  T* Ks = reinterpret_cast<T*>(smem);
  T* Vs = Ks + B * D;
  float* Ss = reinterpret_cast<float*>(Vs + B * D);  // [B][B + 1]

  const int64_t b = ceil_div64(n, B);
  const int64_t i = b - 1 - blockIdx.x;  // longest rows first
  const int h = blockIdx.y, g = h / group;
  const int r = threadIdx.x >> 1, half = threadIdx.x & 1;
  const int64_t t = i * B + r;
  const bool qvalid = t < n;

  float qv[HD], acc[HD];
  const T* qrow = q + h * lay.q.head + (qvalid ? t : 0) * lay.q.tok + half * HD;
#pragma unroll
  for (int c = 0; c < HD; ++c) {
    qv[c] = qvalid ? to_f32(qrow[c]) * qscale : 0.f;
    acc[c] = 0.f;
  }
  float m = -INFINITY, l = 0.f;

  const int32_t* rp = row_ptr + (int64_t)h * (b + 1);
  int32_t e0 = rp[i], e1 = rp[i + 1];
  if (e0 < 0 || e1 < e0 || e1 > nnz) {  // corrupt row pointers: attend to nothing, report
    if (threadIdx.x == 0) record_error(err, GUARD_BAD_CSR);
    e0 = e1 = 0;
  }
  const int32_t* cols = col_idx + (int64_t)h * nnz;
  const T* kh = k + g * lay.k.head;
  const T* vh = v + g * lay.v.head;

  for (int32_t e = e0; e < e1; ++e) {
    const int64_t j = cols[e];
    if (j < 0 || j > i) {  // not a causal block: skip it and report
      if (threadIdx.x == 0) record_error(err, GUARD_BAD_CSR);
      continue;
    }
    __syncthreads();
    const int64_t u0 = j * B;
    const int rows = static_cast<int>(std::min<int64_t>(B, n - u0));
    for (int x = threadIdx.x; x < B * D / VE; x += blockDim.x) {
      const int rr = x / (D / VE), cv = x % (D / VE);
      uint4 kv = make_uint4(0, 0, 0, 0), vv = make_uint4(0, 0, 0, 0);
      if (rr < rows) {
        kv = *reinterpret_cast<const uint4*>(kh + (u0 + rr) * lay.k.tok + cv * VE);
        vv = *reinterpret_cast<const uint4*>(vh + (u0 + rr) * lay.v.tok + cv * VE);
      }
      reinterpret_cast<uint4*>(Ks)[x] = kv;
      reinterpret_cast<uint4*>(Vs)[x] = vv;
    }
    __syncthreads();
    float mb = -INFINITY;
    for (int u = 0; u < B; ++u) {
      const T* kr = Ks + u * D + half * HD;
      float s = 0.f;
#pragma unroll
      for (int c = 0; c < HD; ++c) s = fmaf(qv[c], to_f32(kr[c]), s);
      s += __shfl_xor_sync(0xffffffffu, s, 1);
      const int64_t tu = u0 + u;
      s = (tu < n && tu <= t) ? s : -INFINITY;
      if (half == 0) Ss[r * (B + 1) + u] = s;
      mb = fmaxf(mb, s);
    }
    __syncwarp();
    const float mn = fmaxf(m, mb);
    if (mn == -INFINITY) continue;  // nothing visible yet in this block
    const float corr = exp2f(m - mn);
    l *= corr;
#pragma unroll
    for (int c = 0; c < HD; ++c) acc[c] *= corr;
    for (int u = 0; u < B; ++u) {
      const float p = exp2f(Ss[r * (B + 1) + u] - mn);
      l += p;
      const T* vr = Vs + u * D + half * HD;
#pragma unroll
      for (int c = 0; c < HD; ++c) acc[c] = fmaf(p, to_f32(vr[c]), acc[c]);
    }
    m = mn;
  }
  if (qvalid) {
    const float inv = 1.f / l;
    T* orow = o + h * lay.o.head + t * lay.o.tok + half * HD;
#pragma unroll
    for (int c = 0; c < HD; ++c) orow[c] = from_f32<T>(acc[c] * inv);
  }
}

template <typename T, int D, int B>
cudaError_t launch_t(const sws_handle* h, const void* q, const void* k, const void* v, int64_t n, int32_t hq,
                     int32_t hkv, const PrefillLayout& lay, const int32_t* row_ptr, const int32_t* col_idx, void* o,
                     cudaStream_t st) {
  const size_t smem = 2 * (size_t)B * D * sizeof(T) + (size_t)B * (B + 1) * sizeof(float);
  auto kern = attn_simt_kernel<T, D, B>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int64_t b = ceil_div64(n, B);
  int64_t nnz = 0;
  for (int64_t i = 0; i < b; ++i) nnz += tau_of_row(i, h->cfg.density_num, h->cfg.density_den);
  const float qscale = static_cast<float>(1.4426950408889634 / sqrt((double)D));  // log2(e) / sqrt(d)
  dim3 grid(static_cast<unsigned>(b), hq);
  {
    const cudaError_t le = launch_k(kern, grid, 2 * B, smem, st, static_cast<const T*>(q), static_cast<const T*>(k),
                                    static_cast<const T*>(v), n, hq / hkv, lay, row_ptr, col_idx, nnz, static_cast<T*>(o),
                                    qscale, h->err);
    if (le != cudaSuccess) return le;
  }
  note_launches(1);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_d(const sws_handle* h, const void* q, const void* k, const void* v, int64_t n, int32_t hq,
                     int32_t hkv, const PrefillLayout& lay, const int32_t* rp, const int32_t* ci, void* o,
                     cudaStream_t st) {
  const int d = h->cfg.head_dim, B = h->cfg.block_size;
  if (d == 128 && B == 128) return launch_t<T, 128, 128>(h, q, k, v, n, hq, hkv, lay, rp, ci, o, st);
  if (d == 128 && B == 64) return launch_t<T, 128, 64>(h, q, k, v, n, hq, hkv, lay, rp, ci, o, st);
  if (d == 64 && B == 128) return launch_t<T, 64, 128>(h, q, k, v, n, hq, hkv, lay, rp, ci, o, st);
  return launch_t<T, 64, 64>(h, q, k, v, n, hq, hkv, lay, rp, ci, o, st);
}

}  // namespace

cudaError_t launch_attn_prefill_simt(const sws_handle* h, const void* q, const void* k, const void* v, sws_dtype dt,
                                     int64_t n, int32_t hq, int32_t hkv, const PrefillLayout& lay,
                                     const int32_t* row_ptr, const int32_t* col_idx, void* o, cudaStream_t st) {
  if (dt == SWS_BF16) return launch_d<__nv_bfloat16>(h, q, k, v, n, hq, hkv, lay, row_ptr, col_idx, o, st);
  return launch_d<float>(h, q, k, v, n, hq, hkv, lay, row_ptr, col_idx, o, st);
}

}  // namespace sws
