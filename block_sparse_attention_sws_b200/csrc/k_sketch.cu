// sw_sketch kernels.
//
// "Scout Before You Attend" §3.1 (token-space sketch: block means) and §3.2
// (feature-space sketch: projection by H_d and the sketched block scores
// Q~ K~^T / sqrt(k) under the causal block mask).
//
// 1. pool_mean_kernel: one streaming pass over Q and K (one launch for both).
//    One CTA per SM; each warp walks its own (head, block) items; each item is
//    one contiguous B x d tile fetched by a 1-D bulk copy into the warp's ring
//    of shared-memory stages (mbarrier completion), summed per column (fp32
//    partials over four bf16 rows, fp64 beyond) and scaled by 1 / (rows of the
//    block). HBM-bound: Q and K are read exactly once; the fp64 means go to
//    the workspace.
// 2. project_kernel: q~ = q_bar H_d and k~ = k_bar H_d (b x d x k MACs).
// 3. scores_kernel: S = Q~ K~^T / sqrt(k) on and below the block diagonal.
#include <algorithm>

#include "sws_common.cuh"

namespace sws {
namespace {

// Block means of Q (heads [0, hq)) and K (heads [hq, hq + hkv)):
// means[(head * nblk + blk) * D + c]. Every warp streams its own items through
// a private ring of bulk-copy stages: lane l reads 16-byte vectors l, l + 32,
// ... of the tile, so it always holds the same 16 bytes of columns over a
// strided set of rows; one shuffle level per factor of two finishes the column
// sums, and no CTA-wide barrier is needed.
template <typename T, int D>
__global__ void __launch_bounds__(128) pool_mean_kernel(const T* __restrict__ q, const T* __restrict__ k, int64_t n,
                                                        int32_t hq, int32_t hkv, int32_t B, int64_t nblk,
                                                        double inv_B, double* __restrict__ means, int stages,
                                                        uint32_t stage_bytes, int32_t* err) {
  constexpr int VE = 16 / sizeof(T);  // elements per 16-byte vector
  constexpr int VR = D / VE;          // vectors per row
  static_assert(VR <= 32 && 32 % VR == 0, "row must map onto a whole number of lanes");
  constexpr int LPC = 32 / VR;        // lanes sharing a column group

  extern __shared__ __align__(128) uint8_t smem[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nwarps = blockDim.x >> 5;
  uint8_t* tiles = smem + (size_t)warp * stages * stage_bytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)nwarps * stages * stage_bytes) + warp * 8;

  const int64_t total = (int64_t)(hq + hkv) * nblk;
  const int64_t gw = (int64_t)blockIdx.x * nwarps + warp;  // global warp index
  const int64_t nw = (int64_t)gridDim.x * nwarps;
  const int64_t my_count = gw < total ? (total - gw + nw - 1) / nw : 0;

  auto item_src = [&](int64_t it, uint32_t& bytes) -> const T* {
    const int64_t head = it / nblk, blk = it % nblk;
    const int64_t r0 = blk * B;
    const int64_t rows = (n - r0 < B ? n - r0 : (int64_t)B);
    bytes = static_cast<uint32_t>(rows * D * sizeof(T));
    return head < hq ? q + (head * n + r0) * D : k + ((head - hq) * n + r0) * D;
  };

  if (lane == 0) {
    for (int s = 0; s < stages; ++s) mbar_init(&full[s], 1);
    mbar_fence_init();
    for (int s = 0; s < stages && s < my_count; ++s) {
      uint32_t bytes;
      const T* src = item_src(gw + (int64_t)s * nw, bytes);
      mbar_arrive_expect_tx(&full[s], bytes);
      bulk_g2s(tiles + (size_t)s * stage_bytes, src, bytes, &full[s]);
    }
  }
  __syncwarp();

  const int vc = lane % VR, r_lane = lane / VR;
  for (int64_t m = 0; m < my_count; ++m) {
    const int s = static_cast<int>(m % stages);
    const uint32_t parity = static_cast<uint32_t>((m / stages) & 1);
    if (!__all_sync(0xffffffffu, mbar_wait(&full[s], parity, err))) return;

    const int64_t it = gw + m * nw;
    const int64_t blk = it % nblk;
    const int rows = static_cast<int>(n - blk * B < B ? n - blk * B : (int64_t)B);
    const T* tile = reinterpret_cast<const T*>(tiles + (size_t)s * stage_bytes);

    double acc[VE];
#pragma unroll
    for (int e = 0; e < VE; ++e) acc[e] = 0.0;
    if constexpr (sizeof(T) == 2) {
      // bf16: fp32 partial over groups of four rows, then fp64
      for (int r0 = r_lane; r0 < rows; r0 += 4 * LPC) {
        float part[VE];
#pragma unroll
        for (int e = 0; e < VE; ++e) part[e] = 0.f;
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) {
          const int r = r0 + qq * LPC;
          if (r < rows) {
            const uint4 v = *reinterpret_cast<const uint4*>(tile + (size_t)r * D + vc * VE);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              part[2 * e] += __uint_as_float(w[e] << 16);
              part[2 * e + 1] += __uint_as_float(w[e] & 0xffff0000u);
            }
          }
        }
#pragma unroll
        for (int e = 0; e < VE; ++e) acc[e] += static_cast<double>(part[e]);
      }
    } else {
      for (int r = r_lane; r < rows; r += LPC) {
        const float4 v = *reinterpret_cast<const float4*>(tile + (size_t)r * D + vc * VE);
        acc[0] += v.x;
        acc[1] += v.y;
        acc[2] += v.z;
        acc[3] += v.w;
      }
    }
    __syncwarp();  // every lane is done with the stage
    if (lane == 0 && m + stages < my_count) {
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      uint32_t bytes;
      const T* src = item_src(gw + (m + stages) * nw, bytes);
      mbar_arrive_expect_tx(&full[s], bytes);
      bulk_g2s(tiles + (size_t)s * stage_bytes, src, bytes, &full[s]);
    }
#pragma unroll
    for (int off = VR; off < 32; off <<= 1) {
#pragma unroll
      for (int e = 0; e < VE; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], off);
    }
    if (lane < VR) {
      const double sc = rows == B ? inv_B : 1.0 / rows;
      double* dst = means + it * D + vc * VE;
#pragma unroll
      for (int e = 0; e < VE; e += 2) *reinterpret_cast<double2*>(dst + e) = make_double2(acc[e] * sc, acc[e + 1] * sc);
    }
  }
}

// q~ (rows < q_rows) and k~ from the block means: one warp per (head, block).
// The row of means is held four values per lane and broadcast by shuffles;
// four independent accumulators per output column.
__global__ void __launch_bounds__(256) project_kernel(const double* __restrict__ means, int64_t rows, int64_t q_rows,
                                                      const double* __restrict__ hd, int D, int k,
                                                      double* __restrict__ q_sk, double* __restrict__ k_sk) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (row >= rows) return;
  const double* mr = means + row * D;
  double mv[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) mv[i] = (lane + 32 * i < D) ? mr[lane + 32 * i] : 0.0;
  double* out = row < q_rows ? q_sk + row * k : k_sk + (row - q_rows) * k;
  for (int c0 = 0; c0 < k; c0 += 32) {
    const int c = c0 + lane;
    double a[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      if (32 * g >= D) break;
#pragma unroll 8
      for (int j = 0; j < 32; ++j) {
        const double m = __shfl_sync(0xffffffffu, mv[g], j);
        if (c < k) a[j & 3] = fma(m, hd[(size_t)(32 * g + j) * k + c], a[j & 3]);
      }
    }
    if (c < k) out[c] = (a[0] + a[1]) + (a[2] + a[3]);
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
cudaError_t launch_pool(const sws_handle* h, const T* q, const T* k, int64_t n, int32_t hq, int32_t hkv,
                        double* means, cudaStream_t st) {
  const int32_t B = h->cfg.block_size;
  const int64_t nblk = ceil_div64(n, B);
  const uint32_t stage_bytes = static_cast<uint32_t>(B) * D * sizeof(T);
  // about 192 KB of copies in flight per SM: warps x stages x tile
  const int stages = stage_bytes <= (16u << 10) ? 3 : 2;
  const int warps = std::max(1, std::min(4, static_cast<int>((192u << 10) / (stages * stage_bytes))));
  const size_t smem = (size_t)warps * stages * stage_bytes + (size_t)warps * 8 * sizeof(uint64_t);
  auto kern = pool_mean_kernel<T, D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int64_t total = (int64_t)(hq + hkv) * nblk;
  const int grid = static_cast<int>(std::min<int64_t>(ceil_div64(total, warps), (int64_t)h->num_sms));
  kern<<<grid, warps * 32, smem, st>>>(q, k, n, hq, hkv, B, nblk, 1.0 / B, means, stages, stage_bytes, h->err);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace

size_t sketch_workspace_bytes(const sws_config& c, int64_t n, int32_t hq, int32_t hkv) {
  return (size_t)(hq + hkv) * ceil_div64(n, c.block_size) * c.head_dim * sizeof(double);
}

cudaError_t launch_sketch_means_project(const sws_handle* h, const void* q, const void* k, sws_dtype dt, int64_t n,
                                        int32_t hq, int32_t hkv, double* means, double* q_sk, double* k_sk,
                                        cudaStream_t st) {
  const int d = h->cfg.head_dim;
  cudaError_t e;
  if (dt == SWS_BF16) {
    const auto* pq = static_cast<const __nv_bfloat16*>(q);
    const auto* pk = static_cast<const __nv_bfloat16*>(k);
    e = d == 128 ? launch_pool<__nv_bfloat16, 128>(h, pq, pk, n, hq, hkv, means, st)
                 : launch_pool<__nv_bfloat16, 64>(h, pq, pk, n, hq, hkv, means, st);
  } else {
    const auto* pq = static_cast<const float*>(q);
    const auto* pk = static_cast<const float*>(k);
    e = d == 128 ? launch_pool<float, 128>(h, pq, pk, n, hq, hkv, means, st)
                 : launch_pool<float, 64>(h, pq, pk, n, hq, hkv, means, st);
  }
  if (e != cudaSuccess) return e;
  const int64_t b = ceil_div64(n, h->cfg.block_size);
  const int64_t rows = (int64_t)(hq + hkv) * b;
  project_kernel<<<static_cast<unsigned>(ceil_div64(rows, 8)), 256, 0, st>>>(means, rows, (int64_t)hq * b, h->hd, d,
                                                                             h->cfg.sketch_dim, q_sk, k_sk);
  note_launches(1);
  return cudaGetLastError();
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
