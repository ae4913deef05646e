// sw_walk_select kernels.
//
// "Scout Before You Attend" §4 (sketch-determined walk):
//   A^l  = row softmax of the sketched scores over the causal blocks j <= i,
//   R^0  = (A^0)^s,  R^l = R^{l-1} (A^l)^s,
// then the top-tau key blocks of every row of R^l.
//
// Everything here is fp64: after a few layers the entries of R that decide the
// selection are 1e-20 .. 1e-40 of the row maximum, below what fp32 holds.
// The b x b matrices are lower-triangular, so the GEMM only visits tiles on or
// below the diagonal and, inside a tile pair, only k in [tile(j), tile(i)];
// it runs on the fp64 tensor path.
#include <algorithm>

#include "select.cuh"
#include "sws_common.cuh"

namespace sws {
namespace {

// One warp per row. temp = 1 for the softmax of §4; temp = s gives the
// entrywise power with renormalised rows (softmax(S)^s / sum = softmax(s S)).
// Each lane keeps its exponentials (j = lane + 32 u) in registers between the
// sum and the normalisation, so every entry takes one exponential.
constexpr int kSoftmaxPerLane = 32;  // rows up to 1024 blocks wide

__global__ void __launch_bounds__(256) block_softmax_kernel(const double* __restrict__ S, int64_t b, int64_t rows,
                                                            double temp, double* __restrict__ A) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int64_t i = row % b;
  const double* s = S + row * b;
  double* a = A + row * b;
  double x[kSoftmaxPerLane];
  double mx = -INFINITY;
#pragma unroll
  for (int u = 0; u < kSoftmaxPerLane; ++u) {
    const int64_t j = lane + 32 * u;
    x[u] = j <= i ? temp * s[j] : -INFINITY;
    mx = fmax(mx, x[u]);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  double sum = 0.0;
#pragma unroll
  for (int u = 0; u < kSoftmaxPerLane; ++u) {
    if (32 * u > i) break;  // warp-uniform: no entry j <= i left for any lane
    x[u] = exp(x[u] - mx);  // exp(-inf) = 0 for j > i
    sum += x[u];
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
  const double inv = 1.0 / sum;
#pragma unroll
  for (int u = 0; u < kSoftmaxPerLane; ++u) {
    const int64_t j = lane + 32 * u;
    if (j < b) a[j] = j <= i ? x[u] * inv : 0.0;
  }
}

// The same for rows wider than 32 x kSoftmaxPerLane blocks: two passes over
// the row, the exponentials recomputed for the normalisation.
__global__ void __launch_bounds__(256) block_softmax_wide_kernel(const double* __restrict__ S, int64_t b,
                                                                 int64_t rows, double temp, double* __restrict__ A) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int64_t i = row % b;
  const double* s = S + row * b;
  double* a = A + row * b;
  double mx = -INFINITY;
  for (int64_t j = lane; j <= i; j += 32) mx = fmax(mx, temp * s[j]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  double sum = 0.0;
  for (int64_t j = lane; j <= i; j += 32) sum += exp(temp * s[j] - mx);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
  const double inv = 1.0 / sum;
  for (int64_t j = lane; j < b; j += 32) a[j] = (j <= i) ? exp(temp * s[j] - mx) * inv : 0.0;
}

// C = A * Bm for lower-triangular b x b matrices on the fp64 tensor path
// (mma.sync m16n8k4 f64). One 32 x 32 output tile per CTA of two warps (on or
// below the diagonal, heaviest first; many small CTAs keep every SM busy and
// waste less of the triangle than large tiles), each warp a 16 x 32 slice;
// k staged 16 at a time through padded shared memory (row strides of 20 and
// 36 doubles make the fragment loads conflict-free) with the next chunk
// prefetched into registers. Entries above the diagonal of A and Bm are
// treated as zero whatever the buffers hold.
constexpr int kTT = 32, kTK = 16, kGemmThreads = 64;
constexpr int kApad = kTK + 4;   // A tile row stride (doubles)
constexpr int kBpad = kTT + 4;   // B tile row stride (doubles)

__device__ __forceinline__ void tile_of(int64_t t, int64_t nt, int64_t& ti, int64_t& tj) {
  // heaviest tiles (largest ti - tj) first
  for (int64_t dl = nt - 1; dl >= 0; --dl) {
    const int64_t cnt = nt - dl;
    if (t < cnt) { tj = t; ti = t + dl; return; }
    t -= cnt;
  }
  ti = tj = 0;
}

__device__ __forceinline__ void dmma_16x8x4(double (&c)[4], double a0, double a1, double b0) {
  asm volatile(
      "mma.sync.aligned.m16n8k4.row.col.f64.f64.f64.f64 {%0,%1,%2,%3}, {%4,%5}, {%6}, {%0,%1,%2,%3};"
      : "+d"(c[0]), "+d"(c[1]), "+d"(c[2]), "+d"(c[3])
      : "d"(a0), "d"(a1), "d"(b0));
}

__global__ void __launch_bounds__(kGemmThreads, 8) tri_gemm_kernel(const double* __restrict__ A,
                                                                const double* __restrict__ Bm,
                                                                double* __restrict__ C, int64_t b) {
  constexpr int PER = kTT * kTK / kGemmThreads;  // 8 elements of each operand chunk per thread
  __shared__ __align__(16) double As[2][kTT][kApad];
  __shared__ __align__(16) double Bs[2][kTK][kBpad];
  const int64_t nt = ceil_div64(b, kTT);
  int64_t ti, tj;
  tile_of(blockIdx.x, nt, ti, tj);
  const size_t hoff = (size_t)blockIdx.y * b * b;
  const double* Ah = A + hoff;
  const double* Bh = Bm + hoff;
  double* Ch = C + hoff;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t4 = lane & 3;
  const int64_t i0 = ti * kTT, j0 = tj * kTT;
  const int64_t kbeg = j0, kend = std::min<int64_t>(b, i0 + kTT);

  double ra[PER], rb[PER];
  auto load = [&](int64_t k0) {
#pragma unroll
    for (int q = 0; q < PER; ++q) {
      const int e = tid + q * kGemmThreads;
      // A: element (row e / KC, k e % KC): 16 consecutive threads read one row
      const int64_t ar = i0 + e / kTK, ak = k0 + e % kTK;
      ra[q] = (ar < b && ak < kend && ak <= ar) ? Ah[ar * b + ak] : 0.0;
      // B: element (k e / T, column e % T): a warp reads one row
      const int64_t bk = k0 + e / kTT, bc = j0 + e % kTT;
      rb[q] = (bk < kend && bc < b && bc <= bk) ? Bh[bk * b + bc] : 0.0;
    }
  };
  auto store = [&](int buf) {
#pragma unroll
    for (int q = 0; q < PER; ++q) {
      const int e = tid + q * kGemmThreads;
      As[buf][e / kTK][e % kTK] = ra[q];
      Bs[buf][e / kTT][e % kTT] = rb[q];
    }
  };

  double acc[4][4];
#pragma unroll
  for (int n8 = 0; n8 < 4; ++n8)
#pragma unroll
    for (int v = 0; v < 4; ++v) acc[n8][v] = 0.0;

  int buf = 0;
  load(kbeg);
  store(0);
  __syncthreads();
  for (int64_t k0 = kbeg; k0 < kend; k0 += kTK) {
    const bool more = k0 + kTK < kend;
    if (more) load(k0 + kTK);
#pragma unroll
    for (int ks = 0; ks < kTK / 4; ++ks) {
      const double a0 = As[buf][warp * 16 + g][ks * 4 + t4];
      const double a1 = As[buf][warp * 16 + g + 8][ks * 4 + t4];
      double bf[4];
#pragma unroll
      for (int n8 = 0; n8 < 4; ++n8) bf[n8] = Bs[buf][ks * 4 + t4][n8 * 8 + g];
#pragma unroll
      for (int n8 = 0; n8 < 4; ++n8) dmma_16x8x4(acc[n8], a0, a1, bf[n8]);
    }
    if (more) {
      store(buf ^ 1);
      __syncthreads();
      buf ^= 1;
    }
  }
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    const int64_t i = i0 + warp * 16 + g + 8 * hh;
    if (i >= b) continue;
#pragma unroll
    for (int n8 = 0; n8 < 4; ++n8) {
      const int64_t j = j0 + n8 * 8 + 2 * t4;
      if (j < b) Ch[i * b + j] = acc[n8][2 * hh];
      if (j + 1 < b) Ch[i * b + j + 1] = acc[n8][2 * hh + 1];
    }
  }
}

// One warp per row: copies R's row to the walk state (zeros above the
// diagonal), writes row_ptr, and emits the row's top-tau blocks ascending.
// With G > 1 query heads sharing a selection, a warp takes one row of a
// group: it copies the G heads' rows, selects on their sum (added in head
// order) and writes the same blocks to the CSR row of every head.
__global__ void __launch_bounds__(256) select_kernel(const double* __restrict__ R, int64_t b, int64_t rows,
                                                     int32_t G, int32_t num, int32_t den, int64_t nnz,
                                                     double* __restrict__ walk_state, int32_t* __restrict__ row_ptr,
                                                     int32_t* __restrict__ col_idx, int32_t* err) {
  extern __shared__ __align__(16) uint64_t keys_all[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + warp;
  if (row >= rows) return;
  uint64_t* keys = keys_all + (size_t)warp * b;
  int* hist = reinterpret_cast<int*>(keys_all + (size_t)(blockDim.x >> 5) * b) + warp * 256;
  const int64_t grp = row / b, i = row % b;
  const int64_t h0 = grp * G;  // first head of the row's group
  for (int64_t j = lane; j < b; j += 32) {
    double sum = 0.0;
    for (int q = 0; q < G; ++q) {
      const int64_t off = ((h0 + q) * b + i) * b + j;
      const double x = (j <= i) ? R[off] : 0.0;
      walk_state[off] = x;
      sum = q == 0 ? x : sum + x;
    }
    if (j <= i) keys[j] = order_key(sum);
  }
  int64_t rp = 0;
  for (int64_t q = lane; q < i; q += 32) rp += tau_of_row(q, num, den);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) rp += __shfl_xor_sync(0xffffffffu, rp, off);
  const int tau = tau_of_row(i, num, den);
  if (lane == 0) {
    for (int q = 0; q < G; ++q) {
      row_ptr[(h0 + q) * (b + 1) + i] = static_cast<int32_t>(rp);
      if (i == b - 1) row_ptr[(h0 + q) * (b + 1) + b] = static_cast<int32_t>(rp + tau);
    }
  }
  __syncwarp();
  int32_t* out0 = col_idx + h0 * nnz + rp;
  warp_top_tau8(keys, static_cast<int>(i + 1), tau, out0, hist, err);
  __syncwarp();  // the first head's row is written: the others copy it
  for (int q = 1; q < G; ++q)
    for (int t = lane; t < tau; t += 32) col_idx[(h0 + q) * nnz + rp + t] = out0[t];
}

}  // namespace

cudaError_t launch_block_softmax(const sws_handle* h, const double* scores, int64_t b, int32_t hq, double* A,
                                 cudaStream_t st) {
  const int64_t rows = (int64_t)hq * b;
  const double temp = h->cfg.walk_mode == SWS_WALK_ELEMENTWISE ? (double)h->cfg.walk_power : 1.0;
  if (b <= 32 * kSoftmaxPerLane)
    block_softmax_kernel<<<static_cast<unsigned>(ceil_div64(rows, 8)), 256, 0, st>>>(scores, b, rows, temp, A);
  else
    block_softmax_wide_kernel<<<static_cast<unsigned>(ceil_div64(rows, 8)), 256, 0, st>>>(scores, b, rows, temp, A);
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_tri_gemm(const double* A, const double* Bm, double* C, int64_t b, int32_t hq, cudaStream_t st) {
  const int64_t nt = ceil_div64(b, kTT);
  dim3 grid(static_cast<unsigned>(nt * (nt + 1) / 2), hq);
  tri_gemm_kernel<<<grid, kGemmThreads, 0, st>>>(A, Bm, C, b);
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_select(const sws_handle* h, const double* R, int64_t b, int32_t hq, double* walk_state,
                          int32_t* row_ptr, int32_t* col_idx, cudaStream_t st) {
  const int32_t G = h->cfg.select_group > 1 ? h->cfg.select_group : 1;
  const int64_t rows = (int64_t)(hq / G) * b;
  int warps = static_cast<int>(std::min<int64_t>(8, std::max<int64_t>(1, (160 << 10) / (b * 8))));
  const size_t smem = (size_t)warps * (b * sizeof(uint64_t) + 256 * sizeof(int));
  cudaError_t e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int64_t nnz = 0;
  for (int64_t i = 0; i < b; ++i) nnz += tau_of_row(i, h->cfg.density_num, h->cfg.density_den);
  select_kernel<<<static_cast<unsigned>(ceil_div64(rows, warps)), warps * 32, smem, st>>>(
      R, b, rows, G, h->cfg.density_num, h->cfg.density_den, nnz, walk_state, row_ptr, col_idx, h->err);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace sws
