// sw_sketch kernels.
//
// "Scout Before You Attend" §3.1 (token-space sketch: block means) and §3.2
// (feature-space sketch: projection by H_d and the sketched block scores
// Q~ K~^T / sqrt(k) under the causal block mask).
//
// 1. pool_project_kernel: one streaming pass over Q and K (one launch for
//    both): 16-byte loads of the B rows of each block, per-column sums,
//    the means, and their projection q~ = q_bar H_d, k~ = k_bar H_d as a
//    Walsh-Hadamard transform in registers and shuffles. HBM-bound:
//    Q and K are read exactly once and only the b x k sketches are written.
// 2. scores_kernel: S = Q~ K~^T / sqrt(k) on and below the block diagonal, on
//    the fp64 tensor path.
#include <algorithm>

#include "sws_common.cuh"

namespace sws {
namespace {

// 16 bytes from global memory that this kernel reads exactly once: bypass L1.
__device__ __forceinline__ uint4 ld_stream16(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

constexpr int kPoolWarps = 8;   // warps per CTA
constexpr int kPoolBatch = 16;  // 16-byte loads in flight per lane

// Block means of Q (heads [0, hq)) and K (heads [hq, hq + hkv)) and their
// projection by H_d, in one pass over Q and K. One warp per (head, block)
// item, items dealt round-robin over all warps of the grid; a block is B rows
// of D contiguous elements (rows at the tensor's token stride), so lane l always reads the same 16 bytes of
// columns (vector l mod VR of a row) on rows l / VR, l / VR + 32 / VR, ...,
// kPoolBatch of them in flight at a time. bf16 columns are summed in fp32 over
// one batch of rows, then in fp64; fp32 inputs are summed in fp64 throughout.
// The column sums meet in a shuffle tree that leaves every lane with the sums
// of its columns c = VE (l mod VR) + e. H_d[c][j] = scale sign_c
// (-1)^popcount(c & col_j), so q_bar H_d is a Walsh-Hadamard transform of
// sign * q_bar read at the k sampled indices col_j: butterflies over e in
// registers, then over the lane bits with xor shuffles; lane j fetches
// transform entry col_j and scales it by scale / rows (the mean divides the
// sums by the rows the block holds).
// kDense: Q and K are dense [heads, n, D] (the strides are then compile-time
// constants and the row addressing a shift).
template <typename T, int D, bool kDense>
__global__ void __launch_bounds__(kPoolWarps * 32, 2)
    pool_project_kernel(const T* __restrict__ q, const T* __restrict__ k, int64_t n, int32_t hq, int32_t hkv,
                        HeadTok qs, HeadTok ks, int32_t B, int64_t nblk, const double* __restrict__ sign,
                        const int32_t* __restrict__ col, double scale, int32_t ksk, double* __restrict__ q_sk,
                        double* __restrict__ k_sk) {
  grid_dependency_wait();
  allow_dependents();
  constexpr int VE = 16 / sizeof(T);  // elements per 16-byte vector
  constexpr int VR = D / VE;          // vectors per row
  static_assert(VR <= 32 && 32 % VR == 0, "row must map onto a whole number of lanes");
  constexpr int LPC = 32 / VR;        // rows covered by one warp-wide load

  constexpr int kOut = D / 32;  // output columns per lane at most (k <= D)
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int vc = lane % VR, rl = lane / VR;
  double sg[VE];
#pragma unroll
  for (int e = 0; e < VE; ++e) sg[e] = sign[vc * VE + e];
  int olane[kOut], oel[kOut];  // lane and element holding transform entry col_j, j = lane + 32 t
#pragma unroll
  for (int t = 0; t < kOut; ++t) {
    const int j = lane + 32 * t;
    const int pj = j < ksk ? col[j] : 0;
    olane[t] = pj / VE;
    oel[t] = pj % VE;
  }
  const int64_t total = (int64_t)(hq + hkv) * nblk;
  const int64_t nw = (int64_t)gridDim.x * kPoolWarps;
  for (int64_t it = (int64_t)blockIdx.x * kPoolWarps + warp; it < total; it += nw) {
    const int64_t head = it / nblk, blk = it % nblk;
    const int64_t r0 = blk * B;
    const int rows = static_cast<int>(n - r0 < B ? n - r0 : (int64_t)B);
    const int64_t rs = kDense ? D : (head < hq ? qs.tok : ks.tok);  // elements from one row to the next
    const int64_t hs = kDense ? n * D : (head < hq ? qs.head : ks.head);
    const T* src = (head < hq ? q + head * hs : k + (head - hq) * hs) + r0 * rs + vc * VE;

    double acc[VE];
#pragma unroll
    for (int e = 0; e < VE; ++e) acc[e] = 0.0;
    for (int rb = rl; rb < rows; rb += kPoolBatch * LPC) {
      uint4 v[kPoolBatch];
#pragma unroll
      for (int u = 0; u < kPoolBatch; ++u) {
        const int r = rb + u * LPC;
        v[u] = r < rows ? ld_stream16(src + r * rs) : make_uint4(0u, 0u, 0u, 0u);
      }
      if constexpr (sizeof(T) == 2) {
        float part[VE];
#pragma unroll
        for (int e = 0; e < VE; ++e) part[e] = 0.f;
#pragma unroll
        for (int u = 0; u < kPoolBatch; ++u) {
          const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            part[2 * e] += __uint_as_float(w[e] << 16);
            part[2 * e + 1] += __uint_as_float(w[e] & 0xffff0000u);
          }
        }
#pragma unroll
        for (int e = 0; e < VE; ++e) acc[e] += static_cast<double>(part[e]);
      } else {
#pragma unroll
        for (int u = 0; u < kPoolBatch; ++u) {
          acc[0] += static_cast<double>(__uint_as_float(v[u].x));
          acc[1] += static_cast<double>(__uint_as_float(v[u].y));
          acc[2] += static_cast<double>(__uint_as_float(v[u].z));
          acc[3] += static_cast<double>(__uint_as_float(v[u].w));
        }
      }
    }
#pragma unroll
    for (int off = VR; off < 32; off <<= 1) {
#pragma unroll
      for (int e = 0; e < VE; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], off);
    }
    double v[VE];
#pragma unroll
    for (int e = 0; e < VE; ++e) v[e] = acc[e] * sg[e];
#pragma unroll
    for (int hb = 1; hb < VE; hb <<= 1) {
#pragma unroll
      for (int e = 0; e < VE; ++e) {
        if ((e & hb) == 0) {
          const double a = v[e], b2 = v[e + hb];
          v[e] = a + b2;
          v[e + hb] = a - b2;
        }
      }
    }
#pragma unroll
    for (int hb = 1; hb < VR; hb <<= 1) {
      const bool upper = (lane & hb) != 0;
#pragma unroll
      for (int e = 0; e < VE; ++e) {
        const double u = __shfl_xor_sync(0xffffffffu, v[e], hb);
        v[e] = upper ? u - v[e] : v[e] + u;
      }
    }
    const double f = scale / static_cast<double>(rows);
    double* out = head < hq ? q_sk + it * ksk : k_sk + (it - (int64_t)hq * nblk) * ksk;
#pragma unroll
    for (int t = 0; t < kOut; ++t) {
      if (32 * t >= ksk) break;  // warp-uniform
      double w = 0.0;
#pragma unroll
      for (int e = 0; e < VE; ++e) {
        const double x = __shfl_sync(0xffffffffu, v[e], olane[t]);
        if (oel[t] == e) w = x;
      }
      if (lane + 32 * t < ksk) out[lane + 32 * t] = w * f;
    }
  }
}

// S[h, i, j] = q~_i . k~_j / sqrt(k) for j <= i, fp64, on the fp64 tensor path
// (mma.sync m16n8k4 f64): one 32 x 32 tile on or below the block diagonal per
// CTA of two warps (each a 16 x 32 slice). The sketch dimension is staged 32
// at a time (all of it at k = 32: one round of loads) by cp.async straight
// into shared memory, both operands row-major with a row stride of 36
// doubles, which puts every fragment load at the minimum of two wavefronts.
// Eight CTAs fit per SM, so a layer's tiles run in one wave. Query head h
// reads the sketches of KV head h / group.
constexpr int kST = 32, kSC = 32, kSLd = kSC + 4;

__device__ __forceinline__ void dmma_16x8x4_s(double (&c)[4], double a0, double a1, double b0) {
  asm volatile(
      "mma.sync.aligned.m16n8k4.row.col.f64.f64.f64.f64 {%0,%1,%2,%3}, {%4,%5}, {%6}, {%0,%1,%2,%3};"
      : "+d"(c[0]), "+d"(c[1]), "+d"(c[2]), "+d"(c[3])
      : "d"(a0), "d"(a1), "d"(b0));
}

// 8 bytes global -> shared, asynchronously; zero-filled when !valid
__device__ __forceinline__ void cp_async8(void* dst, const void* src, bool valid) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(valid ? 8 : 0)
               : "memory");
}

__global__ void __launch_bounds__(64, 8)
    scores_kernel(const double* __restrict__ q_sk, const double* __restrict__ k_sk, int64_t b, int32_t hq,
                  int32_t group, int32_t k, double inv_sqrt_k, double* __restrict__ S) {
  grid_dependency_wait();
  allow_dependents();
  __shared__ __align__(16) double qs[kST][kSLd];  // [query block][sketch dim]
  __shared__ __align__(16) double ks[kST][kSLd];  // [key block][sketch dim]
  const int64_t t = blockIdx.x;
  // tile (ti, tj), tj <= ti, from the linear lower-triangle index
  int64_t ti = static_cast<int64_t>((sqrt(8.0 * (double)t + 1.0) - 1.0) * 0.5);
  while (ti * (ti + 1) / 2 > t) --ti;
  while ((ti + 1) * (ti + 2) / 2 <= t) ++ti;
  const int64_t tj = t - ti * (ti + 1) / 2;
  const int h = blockIdx.y;
  const double* qh = q_sk + (size_t)h * b * k;
  const double* kh = k_sk + (size_t)(h / group) * b * k;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t4 = lane & 3;
  const int64_t i0 = ti * kST, j0 = tj * kST;
  double acc[4][4];
#pragma unroll
  for (int n8 = 0; n8 < 4; ++n8)
#pragma unroll
    for (int v = 0; v < 4; ++v) acc[n8][v] = 0.0;
  for (int c0 = 0; c0 < k; c0 += kSC) {
    if (c0 > 0) __syncthreads();  // the previous chunk's fragments have been read
#pragma unroll 4
    for (int u = 0; u < kST * kSC / 64; ++u) {
      const int e = tid + 64 * u;
      const int r = e / kSC, c = e % kSC;  // a warp copies one row
      const int64_t qi = i0 + r, kj = j0 + r;
      const bool cok = c0 + c < k;
      cp_async8(&qs[r][c], (qi < b && cok) ? qh + qi * k + c0 + c : qh, qi < b && cok);
      cp_async8(&ks[r][c], (kj < b && cok) ? kh + kj * k + c0 + c : kh, kj < b && cok);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kSC / 4; ++kk) {
      const double a0 = qs[warp * 16 + g][kk * 4 + t4];
      const double a1 = qs[warp * 16 + g + 8][kk * 4 + t4];
#pragma unroll
      for (int n8 = 0; n8 < 4; ++n8) dmma_16x8x4_s(acc[n8], a0, a1, ks[n8 * 8 + g][kk * 4 + t4]);
    }
  }
  const bool pairs = (b & 1) == 0;  // 16-byte aligned row starts
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    const int64_t i = i0 + warp * 16 + g + 8 * hh;
    if (i >= b) continue;
#pragma unroll
    for (int n8 = 0; n8 < 4; ++n8) {
      const int64_t j = j0 + n8 * 8 + 2 * t4;
      double* dst = S + ((size_t)h * b + i) * b + j;
      if (pairs && j + 1 <= i) {
        *reinterpret_cast<double2*>(dst) =
            make_double2(acc[n8][2 * hh] * inv_sqrt_k, acc[n8][2 * hh + 1] * inv_sqrt_k);
      } else {
        if (j <= i) dst[0] = acc[n8][2 * hh] * inv_sqrt_k;
        if (j + 1 <= i) dst[1] = acc[n8][2 * hh + 1] * inv_sqrt_k;
      }
    }
  }
}

template <typename T, int D>
cudaError_t launch_pool_project(const sws_handle* h, const T* q, const T* k, int64_t n, int32_t hq, int32_t hkv,
                                HeadTok qs, HeadTok ks, double* q_sk, double* k_sk, cudaStream_t st) {
  const int32_t B = h->cfg.block_size;
  const int64_t nblk = ceil_div64(n, B);
  const int64_t total = (int64_t)(hq + hkv) * nblk;
  const int grid = static_cast<int>(std::min<int64_t>(ceil_div64(total, kPoolWarps), 2 * (int64_t)h->num_sms));
  const bool dense = qs.tok == D && ks.tok == D && qs.head == n * D && ks.head == n * D;
  {
    const cudaError_t le =
        launch_k(dense ? pool_project_kernel<T, D, true> : pool_project_kernel<T, D, false>, grid, kPoolWarps * 32, 0,
                 st, q, k, n, hq, hkv, qs, ks, B, nblk, h->sign, h->col, h->scale, h->cfg.sketch_dim, q_sk, k_sk);
    if (le != cudaSuccess) return le;
  }
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace

size_t sketch_workspace_bytes(const sws_config&, int64_t, int32_t, int32_t) { return 0; }

cudaError_t launch_sketch_pool_project(const sws_handle* h, const void* q, const void* k, sws_dtype dt, int64_t n,
                                       int32_t hq, int32_t hkv, HeadTok qs, HeadTok ks, double* q_sk, double* k_sk,
                                       cudaStream_t st) {
  const int d = h->cfg.head_dim;
  if (dt == SWS_BF16) {
    const auto* pq = static_cast<const __nv_bfloat16*>(q);
    const auto* pk = static_cast<const __nv_bfloat16*>(k);
    return d == 128 ? launch_pool_project<__nv_bfloat16, 128>(h, pq, pk, n, hq, hkv, qs, ks, q_sk, k_sk, st)
                    : launch_pool_project<__nv_bfloat16, 64>(h, pq, pk, n, hq, hkv, qs, ks, q_sk, k_sk, st);
  }
  const auto* pq = static_cast<const float*>(q);
  const auto* pk = static_cast<const float*>(k);
  return d == 128 ? launch_pool_project<float, 128>(h, pq, pk, n, hq, hkv, qs, ks, q_sk, k_sk, st)
                  : launch_pool_project<float, 64>(h, pq, pk, n, hq, hkv, qs, ks, q_sk, k_sk, st);
}

cudaError_t launch_sketch_scores(const sws_handle* h, const double* q_sk, const double* k_sk, int64_t b, int32_t hq,
                                 int32_t hkv, double* scores, cudaStream_t st) {
  const int64_t nt = ceil_div64(b, kST);
  dim3 grid(static_cast<unsigned>(nt * (nt + 1) / 2), hq);
  const int32_t k = h->cfg.sketch_dim;
  {
    const cudaError_t le = launch_k(scores_kernel, grid, 64, 0, st, q_sk, k_sk, b, hq, hq / hkv, k,
                                    1.0 / sqrt((double)k), scores);
    if (le != cudaSuccess) return le;
  }
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace sws
