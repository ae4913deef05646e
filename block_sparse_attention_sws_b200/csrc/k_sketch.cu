// sw_sketch kernels.
//
// "Scout Before You Attend" §3.1 (token-space sketch: block means) and §3.2
// (feature-space sketch: projection by H_d and the sketched block scores
// Q~ K~^T / sqrt(k) under the causal block mask).
//
// Pool + project: one streaming pass over Q (or K). Persistent CTAs walk the
// (head, block) items; each item is one contiguous B x d tile fetched by a 1-D
// bulk copy into a ring of shared-memory stages (mbarrier completion), summed
// per column (fp32 partials over a few bf16 rows, fp64 beyond), divided by the
// block's row count, and multiplied by H_d. The pass is HBM-bound: Q and K are
// read exactly once.
#include <algorithm>

#include "sws_common.cuh"

namespace sws {
namespace {

constexpr int kPoolThreads = 256;

template <typename T, int D>
__global__ void __launch_bounds__(kPoolThreads) pool_project_kernel(const T* __restrict__ x, int64_t n,
                                                                     int32_t heads, int32_t B, int64_t nblk,
                                                                     const double* __restrict__ hdt, int32_t k,
                                                                     double* __restrict__ out, int stages,
                                                                     uint32_t stage_bytes, int32_t* err) {
  constexpr int VE = 16 / sizeof(T);       // elements per 16-byte vector
  constexpr int VR = D / VE;               // vectors per row
  constexpr int RG = kPoolThreads / VR;    // row groups
  constexpr int NW = kPoolThreads / 32;
  static_assert(VR <= 32 && 32 % VR == 0, "row must map onto a whole number of lanes");

  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* tiles = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)stages * stage_bytes);
  double* red = reinterpret_cast<double*>(full + 8);  // [NW][D]
  double* mean = red + NW * D;                        // [D]

  const int tid = threadIdx.x;
  const int64_t total = (int64_t)heads * nblk;
  if ((int64_t)blockIdx.x >= total) return;
  const int64_t my_count = (total - blockIdx.x + gridDim.x - 1) / gridDim.x;

  auto item_src = [&](int64_t it, uint32_t& bytes) -> const T* {
    const int64_t head = it / nblk, blk = it % nblk;
    const int64_t r0 = blk * B;
    const int64_t rows = (n - r0 < B ? n - r0 : (int64_t)B);
    bytes = static_cast<uint32_t>(rows * D * sizeof(T));
    return x + (head * n + r0) * D;
  };

  if (tid == 0) {
    for (int s = 0; s < stages; ++s) mbar_init(&full[s], 1);
    mbar_fence_init();
  }
  __syncthreads();
  if (tid == 0) {
    for (int s = 0; s < stages && s < my_count; ++s) {
      uint32_t bytes;
      const T* src = item_src(blockIdx.x + (int64_t)s * gridDim.x, bytes);
      mbar_arrive_expect_tx(&full[s], bytes);
      bulk_g2s(tiles + (size_t)s * stage_bytes, src, bytes, &full[s]);
    }
  }

  const int vc = tid % VR, rg = tid / VR;
  const int lane = tid & 31, warp = tid >> 5;
  // projection mapping: P lanes cooperate on one output column c
  int kpad = 1;
  while (kpad < k) kpad <<= 1;
  const int P = min(32, max(1, kPoolThreads / kpad));
  const int pc = tid / P, part = tid % P;

  for (int64_t m = 0; m < my_count; ++m) {
    const int s = static_cast<int>(m % stages);
    const uint32_t parity = static_cast<uint32_t>((m / stages) & 1);
    const bool ok = mbar_wait(&full[s], parity, err);
    if (__syncthreads_or(!ok)) return;

    const int64_t it = blockIdx.x + m * gridDim.x;
    const int64_t blk = it % nblk;
    const int rows = static_cast<int>(n - blk * B < B ? n - blk * B : (int64_t)B);
    const T* tile = reinterpret_cast<const T*>(tiles + (size_t)s * stage_bytes);

    double acc[VE];
#pragma unroll
    for (int e = 0; e < VE; ++e) acc[e] = 0.0;
    if constexpr (sizeof(T) == 2) {
      // bf16: exact-ish fp32 partial over groups of 4 rows, then fp64.
      for (int r0 = rg; r0 < rows; r0 += 4 * RG) {
        float part4[VE];
#pragma unroll
        for (int e = 0; e < VE; ++e) part4[e] = 0.f;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int r = r0 + q * RG;
          if (r < rows) {
            const uint4 v = *reinterpret_cast<const uint4*>(tile + (size_t)r * D + vc * VE);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              part4[2 * e] += __uint_as_float(w[e] << 16);
              part4[2 * e + 1] += __uint_as_float(w[e] & 0xffff0000u);
            }
          }
        }
#pragma unroll
        for (int e = 0; e < VE; ++e) acc[e] += static_cast<double>(part4[e]);
      }
    } else {
      for (int r = rg; r < rows; r += RG) {
        const float4 v = *reinterpret_cast<const float4*>(tile + (size_t)r * D + vc * VE);
        acc[0] += v.x;
        acc[1] += v.y;
        acc[2] += v.z;
        acc[3] += v.w;
      }
    }
    // reduce over the row groups held by this warp (lanes with equal vc)
#pragma unroll
    for (int off = VR; off < 32; off <<= 1) {
#pragma unroll
      for (int e = 0; e < VE; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], off);
    }
    __syncthreads();  // every thread is done with the tile
    if (tid == 0 && m + stages < my_count) {
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      uint32_t bytes;
      const T* src = item_src(blockIdx.x + (m + stages) * gridDim.x, bytes);
      mbar_arrive_expect_tx(&full[s], bytes);
      bulk_g2s(tiles + (size_t)s * stage_bytes, src, bytes, &full[s]);
    }
    if (lane < VR) {
#pragma unroll
      for (int e = 0; e < VE; ++e) red[warp * D + vc * VE + e] = acc[e];
    }
    __syncthreads();
    if (tid < D) {
      double sum = 0.0;
#pragma unroll
      for (int w = 0; w < NW; ++w) sum += red[w * D + tid];
      mean[tid] = sum / rows;
    }
    __syncthreads();
    double pr = 0.0;
    if (pc < k) {
      const double* hrow = hdt + (size_t)pc * D;
      for (int r = part; r < D; r += P) pr += mean[r] * __ldg(hrow + r);
    }
    for (int off = P >> 1; off > 0; off >>= 1) pr += __shfl_xor_sync(0xffffffffu, pr, off);
    if (pc < k && part == 0) out[it * k + pc] = pr;
  }
}

// S[h, i, j] = q~_i . k~_j / sqrt(k) for j <= i, fp64, 64 x 64 tiles on and
// below the diagonal; 256 threads, 4 x 4 outputs each.
constexpr int kST = 64;
constexpr int kSC = 32;  // sketch-dimension chunk staged in shared memory

__global__ void __launch_bounds__(256) scores_kernel(const double* __restrict__ q_sk, const double* __restrict__ k_sk,
                                                     int64_t b, int32_t hq, int32_t group, int32_t k,
                                                     double inv_sqrt_k, double* __restrict__ S) {
  __shared__ double qs[kST][kSC + 1];
  __shared__ double ks[kST][kSC + 1];
  const int64_t t = blockIdx.x;
  // tile (ti, tj), tj <= ti, from the linear lower-triangle index
  int64_t ti = static_cast<int64_t>((sqrt(8.0 * (double)t + 1.0) - 1.0) * 0.5);
  while (ti * (ti + 1) / 2 > t) --ti;
  while ((ti + 1) * (ti + 2) / 2 <= t) ++ti;
  const int64_t tj = t - ti * (ti + 1) / 2;
  const int h = blockIdx.y;
  const int g = h / group;
  const double* qh = q_sk + (size_t)h * b * k;
  const double* kh = k_sk + (size_t)g * b * k;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  double acc[4][4] = {};
  for (int c0 = 0; c0 < k; c0 += kSC) {
    for (int e = threadIdx.x; e < kST * kSC; e += 256) {
      const int r = e / kSC, c = e % kSC;
      const int64_t qi = ti * kST + r, kj = tj * kST + r;
      qs[r][c] = (qi < b && c0 + c < k) ? qh[qi * k + c0 + c] : 0.0;
      ks[r][c] = (kj < b && c0 + c < k) ? kh[kj * k + c0 + c] : 0.0;
    }
    __syncthreads();
#pragma unroll 4
    for (int c = 0; c < kSC; ++c) {
      double a[4], bb[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        a[u] = qs[ty + 16 * u][c];
        bb[u] = ks[tx + 16 * u][c];
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[u][v] = fma(a[u], bb[v], acc[u][v]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int64_t i = ti * kST + ty + 16 * u;
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const int64_t j = tj * kST + tx + 16 * v;
      if (i < b && j <= i) S[((size_t)h * b + i) * b + j] = acc[u][v] * inv_sqrt_k;
    }
  }
}

template <typename T, int D>
cudaError_t launch_pool(const sws_handle* h, const T* x, int64_t n, int32_t heads, double* out, cudaStream_t st) {
  const int32_t B = h->cfg.block_size;
  const int64_t nblk = ceil_div64(n, B);
  const uint32_t stage_bytes = static_cast<uint32_t>(B) * D * sizeof(T);
  const int stages = std::max(2, std::min(6, static_cast<int>((128u << 10) / stage_bytes)));
  const size_t smem = (size_t)stages * stage_bytes + 8 * sizeof(uint64_t) +
                      (size_t)(kPoolThreads / 32 + 1) * D * sizeof(double);
  auto kern = pool_project_kernel<T, D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int per_sm = std::max(1, static_cast<int>((200u << 10) / smem));
  const int64_t total = (int64_t)heads * nblk;
  const int grid = static_cast<int>(std::min<int64_t>(total, (int64_t)h->num_sms * per_sm));
  kern<<<grid, kPoolThreads, smem, st>>>(x, n, heads, B, nblk, h->hdt, h->cfg.sketch_dim, out, stages, stage_bytes,
                                         h->err);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_sketch_pool_project(const sws_handle* h, const void* x, sws_dtype dt, int64_t n, int32_t heads,
                                       double* out, cudaStream_t st) {
  const int d = h->cfg.head_dim;
  if (dt == SWS_BF16) {
    const auto* p = static_cast<const __nv_bfloat16*>(x);
    return d == 128 ? launch_pool<__nv_bfloat16, 128>(h, p, n, heads, out, st)
                    : launch_pool<__nv_bfloat16, 64>(h, p, n, heads, out, st);
  }
  const auto* p = static_cast<const float*>(x);
  return d == 128 ? launch_pool<float, 128>(h, p, n, heads, out, st) : launch_pool<float, 64>(h, p, n, heads, out, st);
}

cudaError_t launch_sketch_scores(const sws_handle* h, const double* q_sk, const double* k_sk, int64_t b, int32_t hq,
                                 int32_t hkv, double* scores, cudaStream_t st) {
  const int64_t nt = ceil_div64(b, kST);
  dim3 grid(static_cast<unsigned>(nt * (nt + 1) / 2), hq);
  const int32_t k = h->cfg.sketch_dim;
  scores_kernel<<<grid, 256, 0, st>>>(q_sk, k_sk, b, hq, hq / hkv, k, 1.0 / sqrt((double)k), scores);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace sws
