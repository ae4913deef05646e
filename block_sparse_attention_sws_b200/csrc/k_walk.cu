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

template <int PL>  // entries per lane: rows up to 32 PL blocks wide
__global__ void __launch_bounds__(256) block_softmax_kernel(const double* __restrict__ S, int64_t b, int64_t rows,
                                                            double temp, double* __restrict__ A) {
  grid_dependency_wait();
  allow_dependents();
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int64_t i = row % b;
  const double* s = S + row * b;
  double* a = A + row * b;
  double x[PL];
  double mx = -INFINITY;
#pragma unroll
  for (int u = 0; u < PL; ++u) {
    const int64_t j = lane + 32 * u;
    x[u] = j <= i ? temp * s[j] : -INFINITY;
    mx = fmax(mx, x[u]);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  double sum = 0.0;
#pragma unroll
  for (int u = 0; u < PL; ++u) {
    if (32 * u > i) break;  // warp-uniform: no entry j <= i left for any lane
    x[u] = exp(x[u] - mx);  // exp(-inf) = 0 for j > i
    sum += x[u];
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
  const double inv = 1.0 / sum;
#pragma unroll
  for (int u = 0; u < PL; ++u) {
    const int64_t j = lane + 32 * u;
    if (j < b) a[j] = j <= i ? x[u] * inv : 0.0;
  }
}

// The same for rows wider than 32 x kSoftmaxPerLane blocks: two passes over
// the row, the exponentials recomputed for the normalisation.
__global__ void __launch_bounds__(256) block_softmax_wide_kernel(const double* __restrict__ S, int64_t b,
                                                                 int64_t rows, double temp, double* __restrict__ A) {
  grid_dependency_wait();
  allow_dependents();
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

// The same row softmax without the sketched scores in memory: each CTA of two
// warps takes one 32-row tile of one head and forms its scores
// S_ij = q~_i . k~_j / sqrt(k), j <= i, itself, 32 key blocks at a time, on the
// fp64 tensor path (mma.sync m16n8k4 f64), from q~ and k~ staged in shared
// memory. Two passes over the row tile's key tiles: the first keeps each row's
// running maximum and sum of exponentials, the second forms the tile's scores
// again and writes exp(temp S - max) / sum. The scores come out of the same
// products in the same order as in scores_kernel, so they are bit for bit the
// ones sws_sketch writes; only the order of the row sum differs from
// block_softmax_kernel. Row tiles run longest first. Entries above the
// diagonal are not written (every reader masks them).
constexpr int kFT = 32;  // rows and key blocks per tile

__device__ __forceinline__ void cp_async8_w(void* dst, const void* src, bool valid) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(valid ? 8 : 0)
               : "memory");
}

// rows r0.. r0 + 31 of a [rows, k] fp64 matrix into a [32][ld] shared tile,
// zero-filled past `rows` and past k up to kpad
__device__ __forceinline__ void stage_tile(double* dst, const double* src, int64_t r0, int64_t rows, int32_t k,
                                           int32_t kpad, int ld, int tid, int nthr) {
  for (int e = tid; e < kFT * kpad; e += nthr) {
    const int r = e / kpad, c = e % kpad;
    const bool ok = r0 + r < rows && c < k;
    cp_async8_w(dst + r * ld + c, ok ? src + (r0 + r) * k + c : src, ok);
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
}

__device__ __forceinline__ void dmma_16x8x4_f(double (&c)[4], double a0, double a1, double b0) {
  asm volatile(
      "mma.sync.aligned.m16n8k4.row.col.f64.f64.f64.f64 {%0,%1,%2,%3}, {%4,%5}, {%6}, {%0,%1,%2,%3};"
      : "+d"(c[0]), "+d"(c[1]), "+d"(c[2]), "+d"(c[3])
      : "d"(a0), "d"(a1), "d"(b0));
}

__global__ void __launch_bounds__(64) sketch_softmax_kernel(const double* __restrict__ q_sk,
                                                            const double* __restrict__ k_sk, int64_t b, int32_t hq,
                                                            int32_t group, int32_t k, int32_t kpad,
                                                            double inv_sqrt_k, double temp, double* __restrict__ A) {
  grid_dependency_wait();
  allow_dependents();
  extern __shared__ __align__(16) double fsm[];
  const int ld = kpad + 4;  // kpad % 32 == 0: fragment loads take the minimum two wavefronts
  double* qs = fsm;                   // [32][ld]
  double* ks0 = fsm + kFT * ld;       // [2][32][ld]
  const int64_t nt = ceil_div64(b, kFT);
  const int64_t ti = nt - 1 - static_cast<int64_t>(blockIdx.x) / hq;  // longest rows first
  const int h = static_cast<int>(blockIdx.x % hq);
  const double* qh = q_sk + (size_t)h * b * k;
  const double* kh = k_sk + (size_t)(h / group) * b * k;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t4 = lane & 3;
  const int64_t i0 = ti * kFT;
  stage_tile(qs, qh, i0, b, k, kpad, ld, tid, 64);
  // this lane's two rows: i0 + 16 warp + g + 8 hh
  double m[2] = {-INFINITY, -INFINITY}, l[2] = {0.0, 0.0};
  for (int pass = 0; pass < 2; ++pass) {
    stage_tile(ks0, kh, 0, b, k, kpad, ld, tid, 64);
    for (int64_t tj = 0; tj <= ti; ++tj) {
      double* ks = ks0 + (tj & 1) * kFT * ld;
      if (tj < ti) {
        stage_tile(ks0 + ((tj + 1) & 1) * kFT * ld, kh, (tj + 1) * kFT, b, k, kpad, ld, tid, 64);
        asm volatile("cp.async.wait_group 1;" ::: "memory");
      } else {
        asm volatile("cp.async.wait_group 0;" ::: "memory");
      }
      __syncthreads();
      double acc[4][4];
#pragma unroll
      for (int n8 = 0; n8 < 4; ++n8)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[n8][v] = 0.0;
      for (int kk = 0; kk < kpad / 4; ++kk) {
        const double a0 = qs[(warp * 16 + g) * ld + kk * 4 + t4];
        const double a1 = qs[(warp * 16 + g + 8) * ld + kk * 4 + t4];
#pragma unroll
        for (int n8 = 0; n8 < 4; ++n8) dmma_16x8x4_f(acc[n8], a0, a1, ks[(n8 * 8 + g) * ld + kk * 4 + t4]);
      }
      const int64_t j0 = tj * kFT;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int64_t i = i0 + warp * 16 + g + 8 * hh;
        double x[8];
#pragma unroll
        for (int n8 = 0; n8 < 4; ++n8)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int64_t j = j0 + n8 * 8 + 2 * t4 + e;
            x[2 * n8 + e] = (i < b && j <= i) ? temp * (acc[n8][2 * hh + e] * inv_sqrt_k) : -INFINITY;
          }
        if (pass == 0) {
          double tm = x[0];
#pragma unroll
          for (int u = 1; u < 8; ++u) tm = fmax(tm, x[u]);
          tm = fmax(tm, __shfl_xor_sync(0xffffffffu, tm, 1));
          tm = fmax(tm, __shfl_xor_sync(0xffffffffu, tm, 2));
          const double mn = fmax(m[hh], tm);
          double sum = 0.0;
          if (mn != -INFINITY) {
#pragma unroll
            for (int u = 0; u < 8; ++u) sum += exp(x[u] - mn);  // exp(-inf) = 0 for masked entries
          }
          sum += __shfl_xor_sync(0xffffffffu, sum, 1);
          sum += __shfl_xor_sync(0xffffffffu, sum, 2);
          if (mn != -INFINITY) {
            l[hh] = l[hh] * exp(m[hh] - mn) + sum;  // exp(-inf) = 0 while nothing was seen
            m[hh] = mn;
          }
        } else if (i < b) {
          const double inv = 1.0 / l[hh];
          double* arow = A + ((size_t)h * b + i) * b;
#pragma unroll
          for (int n8 = 0; n8 < 4; ++n8) {
            const int64_t j = j0 + n8 * 8 + 2 * t4;
            const double v0 = exp(x[2 * n8] - m[hh]) * inv, v1 = exp(x[2 * n8 + 1] - m[hh]) * inv;
            if ((b & 1) == 0 && j + 1 <= i) {
              *reinterpret_cast<double2*>(arow + j) = make_double2(v0, v1);
            } else {
              if (j <= i) arow[j] = v0;
              if (j + 1 <= i) arow[j + 1] = v1;
            }
          }
        }
      }
      __syncthreads();  // every warp is done with this key tile before it is refilled
    }
  }
}

// C = A * Bm for lower-triangular b x b matrices on the fp64 tensor path
// (mma.sync m16n8k4 f64). On this part each SM sub-partition completes one
// such product about every 32 cycles, and one warp with one accumulator chain
// already keeps it busy, so what matters is that every sub-partition always
// has a product to issue and that the loads feeding it stay cheap.
//
// One 32 x 32 output tile (on or below the diagonal) per CTA of four warps.
// The tile's k range, key blocks J..I of the walk, is cut into chunks of 8
// and warp w takes chunks w, w+4, ...: a long tile and a short one alike keep
// all four sub-partitions of their SM equally busy. Each warp reads its
// fragments from L2 straight into registers (every operand element is used by
// exactly one warp, so shared-memory staging would only add traffic), with the
// next chunk's loads in flight while the current chunk's sixteen products
// issue. The loads are 16 bytes wide: a lane takes two neighbouring k of an A
// row and two neighbouring columns of a Bm row, and the k order inside a chunk
// and the column order inside the tile are permuted to match (a sum over k
// does not care about its order up to rounding; the columns are put back when
// the tile is written). The four partial tiles are summed in warp order
// through shared memory, so the result does not depend on scheduling. Tiles
// go out heaviest first across all heads. Entries above the diagonal of A and
// Bm are treated as zero whatever the buffers hold. An odd b (rows not 16-byte
// aligned) and the tiles of the last tile row of a ragged b take a checked
// path with 8-byte loads.
constexpr int kTT = 32, kGemmWarps = 4, kGemmThreads = 32 * kGemmWarps;
constexpr int kPartLd = kTT + 2;  // partial-tile row stride (doubles): 16-B rows, spread banks

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
  asm(
      "mma.sync.aligned.m16n8k4.row.col.f64.f64.f64.f64 {%0,%1,%2,%3}, {%4,%5}, {%6}, {%0,%1,%2,%3};"
      : "+d"(c[0]), "+d"(c[1]), "+d"(c[2]), "+d"(c[3])
      : "d"(a0), "d"(a1), "d"(b0));
}

// One warp's share of a tile: chunks warp, warp + 4, ... of [j0, kend), chunk
// c covering k = j0 + 8c .. j0 + 8c + 7. Lane (g, t4) holds, for the chunk's
// two mma k-steps q = 0, 1, the k = j0 + 8c + 2 t4 + q: A at rows
// i0 + g + 8m (m = 0..3, the two m16 halves), Bm at columns j0 + 16p + 2g + e
// (p, e = 0, 1), which form the n8 block n = 2p + e. So the accumulator
// element v of (h, n) is C[16h + g + 8(v >> 1)][16p + 4 t4 + 2(v & 1) + e].
template <bool kChecked>
__device__ __forceinline__ void tile_products(const double* __restrict__ Ah, const double* __restrict__ Bh, int64_t b,
                                              int64_t i0, int64_t j0, int64_t kend, int warp, int lane,
                                              double (&acc)[2][4][4]) {
  const int g = lane >> 2, t4 = lane & 3;
  const int nchunks = static_cast<int>((kend - j0 + 7) >> 3);
  // coordinates relative to j0 (all fit in 32 bits: b <= 8192)
  const int di = static_cast<int>(i0 - j0), rb = static_cast<int>(b - j0), re = static_cast<int>(kend - j0);
  const double* pa = Ah + (i0 + g) * b + j0 + 2 * t4;    // row i0 + g, column j0 + 2 t4
  const double* pb = Bh + (j0 + 2 * t4) * b + j0 + 2 * g;  // row j0 + 2 t4, column j0 + 2g
  double2 fa[2][4], fb[2][4];  // fb[.][2q + p]
  // raw loads; the masks are applied where the products use the values, so
  // that nothing waits on a load before the previous chunk's products issue
  auto load = [&](int c, double2(&xa)[4], double2(&xb)[4]) {
    const double* a = pa + 8 * c;
    const double* bp = pb + (int64_t)(8 * c) * b;
    const int kr = 8 * c + 2 * t4;  // k - j0 of q = 0
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const double* src = a + (int64_t)(8 * m) * b;
      if (!kChecked) {
        xa[m] = __ldg(reinterpret_cast<const double2*>(src));
      } else {
        const bool row_ok = di + g + 8 * m < rb;
        xa[m].x = (row_ok && kr < re) ? __ldg(src) : 0.0;
        xa[m].y = (row_ok && kr + 1 < re) ? __ldg(src + 1) : 0.0;
      }
    }
#pragma unroll
    for (int q = 0; q < 2; ++q)
#pragma unroll
      for (int p = 0; p < 2; ++p) {
        const double* src = bp + q * b + 16 * p;
        if (!kChecked) {
          xb[2 * q + p] = __ldg(reinterpret_cast<const double2*>(src));
        } else {
          const bool k_ok = kr + q < re;
          const int cr = 16 * p + 2 * g;  // column - j0
          xb[2 * q + p].x = (k_ok && cr < rb) ? __ldg(src) : 0.0;
          xb[2 * q + p].y = (k_ok && cr + 1 < rb) ? __ldg(src + 1) : 0.0;
        }
      }
  };
  auto mma = [&](int c, const double2(&xa)[4], const double2(&xb)[4]) {
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int kr = 8 * c + 2 * t4 + q;
      double ma[4], mb[4];
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const double x = q ? xa[m].y : xa[m].x;
        ma[m] = kr <= di + g + 8 * m ? x : 0.0;  // A above its diagonal
      }
#pragma unroll
      for (int p = 0; p < 2; ++p)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const double x = e ? xb[2 * q + p].y : xb[2 * q + p].x;
          mb[2 * p + e] = 16 * p + 2 * g + e <= kr ? x : 0.0;  // Bm above its diagonal
        }
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int n = 0; n < 4; ++n) dmma_16x8x4(acc[h][n], ma[2 * h], ma[2 * h + 1], mb[n]);
    }
  };
  int c = warp;
  if (c >= nchunks) return;
  load(c, fa[0], fb[0]);
  // two chunks per trip, the loads of the next one in flight under the products of this one
  while (true) {
    const bool more1 = c + kGemmWarps < nchunks;
    if (more1) load(c + kGemmWarps, fa[1], fb[1]);
    mma(c, fa[0], fb[0]);
    if (!more1) break;
    c += kGemmWarps;
    const bool more0 = c + kGemmWarps < nchunks;
    if (more0) load(c + kGemmWarps, fa[0], fb[0]);
    mma(c, fa[1], fb[1]);
    if (!more0) break;
    c += kGemmWarps;
  }
}

__global__ void __launch_bounds__(kGemmThreads, 3) tri_gemm_kernel(const double* __restrict__ A,
                                                                const double* __restrict__ Bm,
                                                                double* __restrict__ C, int64_t b, int32_t hq) {
  grid_dependency_wait();
  allow_dependents();
  __shared__ __align__(16) double part[kGemmWarps][kTT][kPartLd];
  const int64_t nt = ceil_div64(b, kTT);
  const int64_t head = blockIdx.x % hq;  // tile-major: every head's heaviest tile first
  int64_t ti, tj;
  tile_of(blockIdx.x / hq, nt, ti, tj);
  const size_t hoff = (size_t)head * b * b;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t4 = lane & 3;
  const int64_t i0 = ti * kTT, j0 = tj * kTT;
  const int64_t kend = std::min<int64_t>(b, i0 + kTT);
  const bool pairs = (b & 1) == 0;  // 16-B aligned row starts

  double acc[2][4][4];
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int n = 0; n < 4; ++n)
#pragma unroll
      for (int v = 0; v < 4; ++v) acc[h][n][v] = 0.0;
  if (i0 + kTT <= b && pairs)
    tile_products<false>(A + hoff, Bm + hoff, b, i0, j0, kend, warp, lane, acc);
  else
    tile_products<true>(A + hoff, Bm + hoff, b, i0, j0, kend, warp, lane, acc);

  // accumulator element v of (h, n = 2p + e): row 16h + g + 8(v >> 1),
  // column 16p + 4 t4 + 2(v & 1) + e; a lane's four columns of one row are contiguous
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int p = 0; p < 2; ++p)
#pragma unroll
      for (int hv = 0; hv < 2; ++hv) {
        double* dst = &part[warp][16 * h + g + 8 * hv][16 * p + 4 * t4];
        *reinterpret_cast<double2*>(dst) = make_double2(acc[h][2 * p][2 * hv], acc[h][2 * p + 1][2 * hv]);
        *reinterpret_cast<double2*>(dst + 2) =
            make_double2(acc[h][2 * p][2 * hv + 1], acc[h][2 * p + 1][2 * hv + 1]);
      }
  __syncthreads();
  double* Ch = C + hoff;
#pragma unroll
  for (int q = 0; q < kTT * kTT / 2 / kGemmThreads; ++q) {
    const int e2 = tid + q * kGemmThreads;
    const int r = e2 >> 4, c = 2 * (e2 & 15);
    const int64_t i = i0 + r, j = j0 + c;
    if (i >= b) continue;
    double2 sum = *reinterpret_cast<const double2*>(&part[0][r][c]);
#pragma unroll
    for (int w = 1; w < kGemmWarps; ++w) {
      const double2 pw = *reinterpret_cast<const double2*>(&part[w][r][c]);
      sum.x += pw.x;
      sum.y += pw.y;
    }
    if (pairs && j + 1 < b) {
      *reinterpret_cast<double2*>(Ch + i * b + j) = sum;
    } else {
      if (j < b) Ch[i * b + j] = sum.x;
      if (j + 1 < b) Ch[i * b + j + 1] = sum.y;
    }
  }
}

// The same product with 64 x 64 output tiles, for walks of 1024 blocks and more.
//
// One CTA of four warps per tile, four CTAs per SM, operands staged in shared
// memory: the k range of the tile, key blocks J..I, is streamed in steps of 16
// through a double-buffered cp.async ring (a 64 x 16 panel of A and a 16 x 64
// panel of Bm per step). Entries above the diagonals of A and Bm are never
// read: the copies stop at the diagonal and fill the rest of the panel with
// zeros, so the products need no masks. Each warp owns a 32 x 32 quarter of
// the tile for the whole k range (eight independent accumulators, one
// fragment load per product) and skips the k steps outside its own part of
// the triangle, so the executed work is 1.10 x the b^3/3 of the product at
// b = 1024. The panels are padded (A rows 20 doubles, Bm rows 68) so that the
// fragment reads of each half-warp fall in distinct banks. Staging quarters
// the L2 traffic of the 32 x 32 tiles; each element is summed in k order.
constexpr int kW64 = 64, kW64Warps = 4, kW64Threads = 32 * kW64Warps, kW64K = 16, kW64Stages = 2;
constexpr int kW64LdA = kW64K + 4;   // A panel [m][k]
constexpr int kW64LdB = kW64 + 4;    // Bm panel [k][n]
constexpr int kW64StageA = kW64 * kW64LdA, kW64StageB = kW64K * kW64LdB;  // doubles
constexpr size_t kW64Smem = sizeof(double) * kW64Stages * (kW64StageA + kW64StageB);
constexpr int64_t kW64MinB = 1024;  // smaller walks keep the 32 x 32 tiles (more CTAs; faster at b = 512)

__device__ __forceinline__ void cp_async16_n(double* dst, const double* src, int bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(bytes)
               : "memory");
}

template <bool kPairs>
__global__ void __launch_bounds__(kW64Threads, 4) tri_gemm64_kernel(const double* __restrict__ A,
                                                                   const double* __restrict__ Bm,
                                                                   double* __restrict__ C, int64_t b64, int32_t hq) {
  grid_dependency_wait();
  allow_dependents();
  extern __shared__ __align__(16) double w64[];
  const int b = static_cast<int>(b64);  // b <= 8192: every offset inside a head fits in 32 bits
  const int nt = (b + kW64 - 1) / kW64;
  const int64_t head = blockIdx.x % hq;  // tile-major: every head's heaviest tile first
  int64_t ti64, tj64;
  tile_of(blockIdx.x / hq, nt, ti64, tj64);
  const size_t hoff = (size_t)head * b * b;
  const double* Ah = A + hoff;
  const double* Bh = Bm + hoff;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t4 = lane & 3;
  const int i0 = static_cast<int>(ti64) * kW64, j0 = static_cast<int>(tj64) * kW64;
  const int kend = min(b, i0 + kW64);
  const int nsteps = (kend - j0 + kW64K - 1) / kW64K;

  auto load = [&](int st, int slot) {
    double* sa = w64 + slot * (kW64StageA + kW64StageB);
    double* sb = sa + kW64StageA;
    const int k0 = j0 + kW64K * st;
    if (kPairs) {
#pragma unroll
      for (int x = 0; x < 4; ++x) {  // A: 64 rows x 8 pairs; A[i][k] is read for k <= i < b
        const int piece = tid + x * kW64Threads;
        const int m = piece >> 3, pr = piece & 7;
        const int i = i0 + m, k = k0 + 2 * pr;
        const int n = i < b ? min(max(i - k + 1, 0), 2) : 0;
        cp_async16_n(sa + m * kW64LdA + 2 * pr, n ? Ah + i * b + k : Ah, 8 * n);
      }
#pragma unroll
      for (int x = 0; x < 4; ++x) {  // Bm: 16 rows x 32 pairs; Bm[k][j] is read for j <= k < b
        const int piece = tid + x * kW64Threads;
        const int kk = piece >> 5, pr = piece & 31;
        const int k = k0 + kk, j = j0 + 2 * pr;
        const int n = k < b ? min(max(k - j + 1, 0), 2) : 0;
        cp_async16_n(sb + kk * kW64LdB + 2 * pr, n ? Bh + k * b + j : Bh, 8 * n);
      }
    } else {
#pragma unroll
      for (int x = 0; x < 8; ++x) {  // A: 64 rows x 16
        const int e = tid + x * kW64Threads;
        const int m = e >> 4, kk = e & 15;
        const int i = i0 + m, k = k0 + kk;
        const bool ok = i < b && k <= i;
        cp_async8_w(sa + m * kW64LdA + kk, ok ? Ah + i * b + k : Ah, ok);
      }
#pragma unroll
      for (int x = 0; x < 8; ++x) {  // Bm: 16 rows x 64
        const int e = tid + x * kW64Threads;
        const int kk = e >> 6, c = e & 63;
        const int k = k0 + kk, j = j0 + c;
        const bool ok = k < b && j <= k;
        cp_async8_w(sb + kk * kW64LdB + c, ok ? Bh + k * b + j : Bh, ok);
      }
    }
  };

  const int wm = warp >> 1, wn = warp & 1;
  const int r0 = 32 * wm, c0 = 32 * wn;  // the warp's 32 x 32 part of the tile
  // the warp's k range: Bm is zero below its first column, A past its last row
  const int wk_lo = j0 + c0, wk_hi = i0 + r0 + 31;
  double acc[2][4][4];
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int n = 0; n < 4; ++n)
#pragma unroll
      for (int v = 0; v < 4; ++v) acc[h][n][v] = 0.0;

  load(0, 0);
  asm volatile("cp.async.commit_group;" ::: "memory");
  for (int st = 0; st < nsteps; ++st) {
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    __syncthreads();
    if (st + 1 < nsteps) load(st + 1, (st + 1) & 1);
    asm volatile("cp.async.commit_group;" ::: "memory");
    const double* sa = w64 + (st & 1) * (kW64StageA + kW64StageB);
    const double* sb = sa + kW64StageA;
    const int k0 = j0 + kW64K * st;
#pragma unroll
    for (int q = 0; q < kW64K / 4; ++q) {
      const int k = k0 + 4 * q;
      if (k + 3 < wk_lo || k > wk_hi) continue;  // all four k of the step are zero for this warp
      double fa[2][2], fb[4];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        fa[h][0] = sa[(r0 + 16 * h + g) * kW64LdA + 4 * q + t4];
        fa[h][1] = sa[(r0 + 16 * h + g + 8) * kW64LdA + 4 * q + t4];
      }
#pragma unroll
      for (int n = 0; n < 4; ++n) fb[n] = sb[(4 * q + t4) * kW64LdB + c0 + 8 * n + g];
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int n = 0; n < 4; ++n) dmma_16x8x4(acc[h][n], fa[h][0], fa[h][1], fb[n]);
    }
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");

  // accumulator element v of (h, n): row r0 + 16h + g + 8(v >> 1), column c0 + 8n + 2 t4 + (v & 1)
  double* Ch = C + hoff;
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int hv = 0; hv < 2; ++hv) {
      const int i = i0 + r0 + 16 * h + g + 8 * hv;
      if (i >= b) continue;
#pragma unroll
      for (int n = 0; n < 4; ++n) {
        const int j = j0 + c0 + 8 * n + 2 * t4;
        const double x0 = acc[h][n][2 * hv], x1 = acc[h][n][2 * hv + 1];
        if (kPairs && j + 1 < b) {
          *reinterpret_cast<double2*>(Ch + (int64_t)i * b + j) = make_double2(x0, x1);
        } else {
          if (j < b) Ch[(int64_t)i * b + j] = x0;
          if (j + 1 < b) Ch[(int64_t)i * b + j + 1] = x1;
        }
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
  grid_dependency_wait();
  allow_dependents();
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

// select_kernel for rows of at most 32 PL blocks: the row is loaded into
// registers with all its loads in flight before its keys go to shared memory
// for the radix select, and the row's CSR offset is summed in 32-bit
// arithmetic when it fits.
template <int PL>
__global__ void __launch_bounds__(256) select_reg_kernel(const double* __restrict__ R, int64_t b, int64_t rows,
                                                         int32_t G, int32_t num, int32_t den, int64_t nnz, int tau32,
                                                         double* __restrict__ walk_state, int32_t* __restrict__ row_ptr,
                                                         int32_t* __restrict__ col_idx, int32_t* err) {
  grid_dependency_wait();
  allow_dependents();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + warp;
  if (row >= rows) return;
  const int64_t grp = row / b, i = row % b;
  const int64_t h0 = grp * G;  // first head of the row's group
  extern __shared__ __align__(16) uint64_t keys_all[];
  uint64_t* keys = keys_all + (size_t)warp * b;
  int* hist = reinterpret_cast<int*>(keys_all + (size_t)(blockDim.x >> 5) * b) + warp * 256;
  double sum[PL];
  for (int q = 0; q < G; ++q) {
    const int64_t off = ((h0 + q) * b + i) * b;
    double x[PL];
#pragma unroll
    for (int u = 0; u < PL; ++u) {
      const int64_t j = lane + 32 * u;
      x[u] = j <= i ? R[off + j] : 0.0;
    }
#pragma unroll
    for (int u = 0; u < PL; ++u) {
      const int64_t j = lane + 32 * u;
      if (j < b) walk_state[off + j] = x[u];
      sum[u] = q == 0 ? x[u] : sum[u] + x[u];
    }
  }
#pragma unroll
  for (int u = 0; u < PL; ++u) {
    const int64_t j = lane + 32 * u;
    if (j <= i) keys[j] = order_key(sum[u]);
  }
  // the CSR offset of row i: the sum of tau over the rows before it, in
  // 32-bit arithmetic when b * num + den fits (the launcher checks)
  int64_t rp = 0;
  if (tau32) {
    uint32_t r32 = 0;
    for (uint32_t q = lane; q < static_cast<uint32_t>(i); q += 32)
      r32 += ((q + 1u) * static_cast<uint32_t>(num) + static_cast<uint32_t>(den) - 1u) / static_cast<uint32_t>(den);
    rp = __reduce_add_sync(0xffffffffu, r32);
  } else {
    for (int64_t q = lane; q < i; q += 32) rp += tau_of_row(q, num, den);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) rp += __shfl_xor_sync(0xffffffffu, rp, off);
  }
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
  const unsigned grid = static_cast<unsigned>(ceil_div64(rows, 8));
  // the fewest registers per lane that hold a row: more warps per SM
  auto kern = b <= 256 ? block_softmax_kernel<8>
              : b <= 512 ? block_softmax_kernel<16>
              : b <= 32 * kSoftmaxPerLane ? block_softmax_kernel<kSoftmaxPerLane>
                                          : block_softmax_wide_kernel;
  {
    const cudaError_t le = launch_k(kern, grid, 256, 0, st, scores, b, rows, temp, A);
    if (le != cudaSuccess) return le;
  }
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_sketch_softmax(const sws_handle* h, const double* q_sk, const double* k_sk, int64_t b, int32_t hq,
                                  int32_t hkv, double* A, cudaStream_t st) {
  const int32_t k = h->cfg.sketch_dim;
  const int32_t kpad = static_cast<int32_t>(ceil_div64(k, 32) * 32);
  const double temp = h->cfg.walk_mode == SWS_WALK_ELEMENTWISE ? (double)h->cfg.walk_power : 1.0;
  const int64_t nt = ceil_div64(b, kFT);
  const size_t smem = 3 * kFT * (kpad + 4) * sizeof(double);
  const cudaError_t ea =
      cudaFuncSetAttribute(sketch_softmax_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (ea != cudaSuccess) return ea;
  {
    const cudaError_t le = launch_k(sketch_softmax_kernel, static_cast<unsigned>(nt * hq), 64, smem, st, q_sk, k_sk, b,
                                    hq, hq / hkv, k, kpad, 1.0 / sqrt((double)k), temp, A);
    if (le != cudaSuccess) return le;
  }
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_tri_gemm(const double* A, const double* Bm, double* C, int64_t b, int32_t hq, cudaStream_t st) {
  if (b >= kW64MinB) {
    const int64_t nt = ceil_div64(b, kW64);
    const int64_t ctas = nt * (nt + 1) / 2 * hq;
    if (ctas > 0x7fffffff) return cudaErrorInvalidValue;
    auto kern = (b & 1) == 0 ? tri_gemm64_kernel<true> : tri_gemm64_kernel<false>;
    const cudaError_t ea = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kW64Smem);
    if (ea != cudaSuccess) return ea;
    const cudaError_t le = launch_k(kern, static_cast<unsigned>(ctas), kW64Threads, kW64Smem, st, A, Bm, C, b, hq);
    if (le != cudaSuccess) return le;
    note_launches(1);
    return cudaGetLastError();
  }
  const int64_t nt = ceil_div64(b, kTT);
  const int64_t ctas = nt * (nt + 1) / 2 * hq;  // one CTA per tile
  if (ctas > 0x7fffffff) return cudaErrorInvalidValue;
  {
    const cudaError_t le = launch_k(tri_gemm_kernel, static_cast<unsigned>(ctas), kGemmThreads, 0, st, A, Bm, C, b, hq);
    if (le != cudaSuccess) return le;
  }
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_select(const sws_handle* h, const double* R, int64_t b, int32_t hq, double* walk_state,
                          int32_t* row_ptr, int32_t* col_idx, cudaStream_t st) {
  const int32_t G = h->cfg.select_group > 1 ? h->cfg.select_group : 1;
  const int64_t rows = (int64_t)(hq / G) * b;
  int64_t nnz = 0;
  for (int64_t i = 0; i < b; ++i) nnz += tau_of_row(i, h->cfg.density_num, h->cfg.density_den);
  if (b <= 1024) {  // the row fits in registers
    auto kern = b <= 256 ? select_reg_kernel<8> : b <= 512 ? select_reg_kernel<16> : select_reg_kernel<32>;
    const size_t smem = 8 * (b * sizeof(uint64_t) + 256 * sizeof(int));
    const cudaError_t ea = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (ea != cudaSuccess) return ea;
    // every tau and the row sums fit in 32 bits: (b + 1) num + den and nnz below 2^32
    const int tau32 = ((b + 1) * (int64_t)h->cfg.density_num + h->cfg.density_den < (int64_t(1) << 32) &&
                       nnz < (int64_t(1) << 32))
                          ? 1
                          : 0;
    const cudaError_t le = launch_k(kern, static_cast<unsigned>(ceil_div64(rows, 8)), 256, smem, st, R, b, rows, G,
                                    h->cfg.density_num, h->cfg.density_den, nnz, tau32, walk_state, row_ptr, col_idx,
                                    h->err);
    if (le != cudaSuccess) return le;
    note_launches(1);
    return cudaGetLastError();
  }
  int warps = static_cast<int>(std::min<int64_t>(8, std::max<int64_t>(1, (160 << 10) / (b * 8))));
  const size_t smem = (size_t)warps * (b * sizeof(uint64_t) + 256 * sizeof(int));
  cudaError_t e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  {
    const cudaError_t le = launch_k(select_kernel, static_cast<unsigned>(ceil_div64(rows, warps)), warps * 32, smem, st,
                                    R, b, rows, G, h->cfg.density_num, h->cfg.density_den, nnz, walk_state, row_ptr,
                                    col_idx, h->err);
    if (le != cudaSuccess) return le;
  }
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace sws
