// Exact decode walk for contexts of any length: the newest query block's row of
// the prefill recurrence of "Scout Before You Attend" §4,
//   R^l[i] = R^{l-1}[i] (A^l)^s,  R^0[i] = e_i (A^0)^s,
// with the rows of each layer's block attention A^l kept in device memory
// between steps instead of being formed again in shared memory.
//
// Row m of A^l (the causal row softmax of q~_m . k~_j / sqrt(k), j <= m) only
// changes while block m is the newest, partial block: rows of complete query
// blocks are fixed once written. So each step writes the newest row alone and
// the s products u <- u A read the rows, which the caller keeps per layer and
// (sequence, query head) as a padded lower triangle: row m holds columns
// 0..m and is padded with zeros to a multiple of four entries, at entry offset
// 4 (q + 1)(2q + r) with q = m div 4, r = m mod 4. Every entry is the rounded
// high word of its fp64 value (sign, 11-bit exponent, 20-bit mantissa), as in
// the shared-memory walk of k_decode_exact.cu, whose scores and softmax the
// rows here reproduce operation for operation.
//
// Per layer and step three launches:
//  1. exact_append_rows_kernel, one CTA per (sequence, KV head): append the
//     token, update the key and query block sums and the newest block's k~
//     and q~, then write the newest row of A for each query head of the group;
//  2. exact_walk_kernel, one CTA per (sequence, query head): u <- u A^s in one
//     sweep over the rows per eight levels of s, from the newest block up to
//     block 0 in blocks of 32 rows. Shared memory holds the partial sums of
//     every column for the eight levels. One warp resolves the 32 x 32
//     diagonal block of a row block level by level, after adding the block
//     below it; the other warps add the block's rows to the columns left of it
//     on the fp64 tensor path. Each entry of the rows is read once per sweep;
//  3. exact_select_kernel, one CTA per (sequence, KV head): the top-tau of
//     each head's row (or one choice for the group) and the union.
#include <algorithm>

#include "select.cuh"
#include "sws_common.cuh"

namespace sws {
namespace {

// entry offset of row m of the padded triangle (rows of 4-entry multiples)
__host__ __device__ __forceinline__ int64_t rows_offset(int64_t m) {
  const int64_t q = m >> 2, r = m & 3;
  return 4 * (q + 1) * (2 * q + r);
}

__device__ __forceinline__ uint32_t hi20(double x) {
  const uint64_t b = static_cast<uint64_t>(__double_as_longlong(x)) + 0x80000000ull;
  return static_cast<uint32_t>(b >> 32);
}
__device__ __forceinline__ double from_hi(uint32_t h) { return __hiloint2double(static_cast<int>(h), 0); }

constexpr int kRowThreads = 256;  // 8 warps
constexpr int kRowWarps = kRowThreads / 32;
constexpr int kMaxK = 32;         // sketch dims (fp32) a row's dot product holds

// Rows [r0, r1) of the block attention of every head of one (sequence, KV
// head) group. qsk: q~ of the group's first head, heads max_blocks * k apart;
// ksk: k~ of the KV head; out: the rows of the group's first head, heads
// rows_offset(max_blocks) entries apart. Scores in fp32 (k~ staged 32 columns
// at a time in shared memory), then per row the maximum, the exponentials, their
// sum in fp64 and the normalisation; each row is written by one warp, its
// padding entries as zeros.
__device__ void build_rows(const double* __restrict__ qsk, const double* __restrict__ ksk, int64_t max_blocks,
                           int k, int group, int r0, int r1, uint32_t* __restrict__ out, float inv_sqrt_k,
                           float* sm) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nr = r1 - r0, npairs = group * nr;
  const int kp = k + 1;
  float* ktile = sm;              // [32][k + 1]
  float* qrows = sm + 32 * kp;    // [npairs][k]
  for (int x = tid; x < npairs * k; x += kRowThreads) {
    const int p = x / k, c = x % k;
    const int hl = p / nr, m = r0 + p % nr;
    qrows[x] = static_cast<float>(qsk[((int64_t)hl * max_blocks + m) * k + c]);
  }
  const int64_t hstride = rows_offset(max_blocks);
  const int ntiles = (r1 - 1) / 32 + 1;
  for (int J = 0; J < ntiles; ++J) {
    __syncthreads();  // the previous tile has been read (and qrows written)
    for (int x = tid; x < 32 * k; x += kRowThreads) {
      const int jj = x / k, c = x % k;
      const int64_t j = 32 * J + jj;
      ktile[jj * kp + c] = j < r1 ? static_cast<float>(ksk[j * k + c]) : 0.f;
    }
    __syncthreads();
    for (int p = warp; p < npairs; p += kRowWarps) {
      const int hl = p / nr, m = r0 + p % nr;
      const int j = 32 * J + lane;
      if (32 * J > m) continue;  // warp-uniform
      const float* qr = qrows + p * k;
      const float* kr = ktile + lane * kp;
      float sdot = 0.f;
      for (int c = 0; c < k; ++c) sdot = fmaf(qr[c], kr[c], sdot);
      if (j <= m) out[hl * hstride + rows_offset(m) + j] = __float_as_uint(sdot * inv_sqrt_k);
    }
  }
  // per row: the softmax over j <= m, by the warp that wrote the row's scores
  for (int p = warp; p < npairs; p += kRowWarps) {
    const int hl = p / nr, m = r0 + p % nr;
    uint32_t* row = out + hl * hstride + rows_offset(m);
    float mx = -INFINITY;
    for (int j = lane; j <= m; j += 32) mx = fmaxf(mx, __uint_as_float(row[j]));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    double se = 0.0;
    for (int j = lane; j <= m; j += 32) {
      const float e = expf(__uint_as_float(row[j]) - mx);
      row[j] = __float_as_uint(e);
      se += static_cast<double>(e);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) se += __shfl_xor_sync(0xffffffffu, se, off);
    const double inv = 1.0 / se;
    const int pitch = ((m + 1) + 3) & ~3;
    for (int j = lane; j < pitch; j += 32)
      row[j] = j <= m ? hi20(static_cast<double>(__uint_as_float(row[j])) * inv) : 0u;
  }
}

__host__ __device__ inline size_t rows_smem_bytes(int k, int group, int rows_per_cta) {
  return (static_cast<size_t>(32) * (k + 1) + static_cast<size_t>(group) * rows_per_cta * k) * sizeof(float);
}

// Rows [32 y, 32 y + 32) (below each sequence's block count) of every head of
// one (sequence, KV head), from the sketches sws_decode_init_cache built.
__global__ void __launch_bounds__(kRowThreads) exact_rows_init_kernel(
    const double* __restrict__ q_sketch, const double* __restrict__ k_sketch, int32_t hq, int32_t hkv,
    int64_t max_len, int64_t max_blocks, const int32_t* __restrict__ seq_lens, int32_t B, int32_t k,
    uint32_t* __restrict__ rows, int32_t* err) {
  grid_dependency_wait();
  allow_dependents();
  extern __shared__ __align__(16) float rsm[];
  const int64_t unit = blockIdx.x;
  const int bi = static_cast<int>(unit / hkv), g = static_cast<int>(unit % hkv);
  const int group = hq / hkv;
  const int32_t len = seq_lens[bi];
  if (len < 1 || len > max_len) {
    if (threadIdx.x == 0) record_error(err, GUARD_BAD_LEN);
    return;
  }
  const int nb = static_cast<int>((len - 1) / B + 1);
  const int r0 = 32 * blockIdx.y;
  if (r0 >= nb) return;
  const int r1 = std::min(nb, r0 + 32);
  const int64_t h0 = (int64_t)bi * hq + (int64_t)g * group;
  build_rows(q_sketch + h0 * max_blocks * k, k_sketch + unit * max_blocks * k, max_blocks, k, group, r0, r1,
             rows + h0 * rows_offset(max_blocks), static_cast<float>(1.0 / sqrt(static_cast<double>(k))), rsm);
}

// Step part 1: append the token; the key and query sums of the newest block, its
// k~ and (per query head of the group) q~; then the newest row of every head.
template <int D>
__global__ void __launch_bounds__(kRowThreads) exact_append_rows_kernel(
    const __nv_bfloat16* __restrict__ q_tok, const __nv_bfloat16* __restrict__ k_tok,
    const __nv_bfloat16* __restrict__ v_tok, int32_t hq, int32_t hkv, int64_t max_len, int64_t max_blocks,
    const int32_t* __restrict__ seq_lens, __nv_bfloat16* __restrict__ k_cache, __nv_bfloat16* __restrict__ v_cache,
    double* __restrict__ k_psum, double* __restrict__ k_sketch, double* __restrict__ q_psum,
    double* __restrict__ q_sketch, const double* __restrict__ hdt, int32_t k, int32_t B, uint32_t* __restrict__ rows,
    int32_t* err) {
  grid_dependency_wait();
  allow_dependents();
  extern __shared__ __align__(16) float rsm[];
  const int group = hq / hkv;
  double* mean = reinterpret_cast<double*>(rsm + (rows_smem_bytes(k, group, 1) + 15) / 16 * 4);  // [D]
  double* qrow = mean + D;                                                                      // [group][D]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t unit = blockIdx.x;
  const int bi = static_cast<int>(unit / hkv), g = static_cast<int>(unit % hkv);
  const int32_t len = seq_lens[bi];
  if (len < 1 || len > max_len) {
    if (tid == 0) record_error(err, GUARD_BAD_LEN);
    return;
  }
  const int64_t pos = len - 1;
  const int i = static_cast<int>(pos / B);
  const int cnt = static_cast<int>(pos % B) + 1;
  if (tid < D) {
    const __nv_bfloat16 kt = k_tok[unit * D + tid];
    k_cache[(unit * max_len + pos) * D + tid] = kt;
    v_cache[(unit * max_len + pos) * D + tid] = v_tok[unit * D + tid];
    double ps = (cnt == 1) ? 0.0 : k_psum[unit * D + tid];
    ps += static_cast<double>(__bfloat162float(kt));
    k_psum[unit * D + tid] = ps;
    mean[tid] = ps / cnt;
  }
  for (int x = tid; x < group * D; x += kRowThreads) {
    const int64_t h = (int64_t)g * group + x / D;
    const int c = x % D;
    const int64_t qi = ((int64_t)bi * hq + h) * D + c;
    double ps = (cnt == 1) ? 0.0 : q_psum[qi];
    ps += static_cast<double>(__bfloat162float(q_tok[qi]));
    q_psum[qi] = ps;
    qrow[x] = ps / cnt;
  }
  __syncthreads();
  double* ksk = k_sketch + unit * max_blocks * k;
  const int64_t h0 = (int64_t)bi * hq + (int64_t)g * group;
  for (int o = warp; o < (group + 1) * k; o += kRowWarps) {
    const int r = o / k, c = o % k;  // r == group: the key block
    const double v = warp_dot_hdt<D>(r == group ? mean : qrow + r * D, hdt + (size_t)c * D, lane);
    if (lane == 0) {
      if (r == group) ksk[(int64_t)i * k + c] = v;
      else q_sketch[((h0 + r) * max_blocks + i) * k + c] = v;
    }
  }
  __syncthreads();  // the sketches written above are read back below
  build_rows(q_sketch + h0 * max_blocks * k, ksk, max_blocks, k, group, i, i + 1,
             rows + h0 * rows_offset(max_blocks), static_cast<float>(1.0 / sqrt(static_cast<double>(k))), rsm);
}

// Step part 2: u <- u A^s for one (sequence, query head), one sweep over the
// stored rows per kLevels levels. Rows go in blocks of 32 from the newest
// block up to block 0. For the columns j left of a block, part[l][j] gathers
// sum over the rows m of the blocks below of u_l[m] A[m][j] (shared memory,
// all levels). Per block M, between two barriers:
//  * warp 0 adds block M's rows to the 32 columns of block M - 32 and then
//    resolves block M - 32's diagonal triangle level by level: u_{l+1}[m] =
//    part[l][m] + sum over the block's rows m' >= m of u_l[m'] A[m'][m],
//    publishing u_0 .. u_{L-1} of its rows for the next block's updates;
//  * warp 1 loads what the chain reads at the next block (a row block's 32 x 32
//    piece and the next triangle) into shared memory, into buffers of
//    alternating parity, sixteen rows at a time, and pulls the rows of
//    the blocks two ahead into L2;
//  * warps 2-15 add block M's rows to every column left of block M - 32,
//    16 columns a warp at a time on the fp64 tensor path (the 8 levels are the
//    n of an m16n8k4 product, the block's rows its k), the next chunk's rows
//    loaded while the current chunk's products run, then one update of part.
// So the chain through the diagonal runs beside the bulk of the row reads,
// and every stored entry is read once per sweep, in a fixed order.
constexpr int kLevels = 8;        // levels of the product per sweep over the rows
constexpr int kWalkThreads = 512;
constexpr int kWalkWarps = kWalkThreads / 32;

__device__ __forceinline__ void dmma_16x8x4(double (&c)[4], double a0, double a1, double b0) {
  asm volatile(
      "mma.sync.aligned.m16n8k4.row.col.f64.f64.f64.f64 {%0,%1,%2,%3}, {%4,%5}, {%6}, {%0,%1,%2,%3};"
      : "+d"(c[0]), "+d"(c[1]), "+d"(c[2]), "+d"(c[3])
      : "d"(a0), "d"(a1), "d"(b0));
}

// Pulls `bytes` (a multiple of 16, from a 16-byte aligned address) into L2; no registers, no completion.
__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

__global__ void __launch_bounds__(kWalkThreads, 1) exact_walk_kernel(
    const uint32_t* __restrict__ rows, int64_t max_len, int64_t max_blocks, const int32_t* __restrict__ seq_lens,
    int32_t B, int32_t hq, int first_layer, int32_t s_pow, double* __restrict__ walk_state, int32_t* err) {
  grid_dependency_wait();
  allow_dependents();
  extern __shared__ __align__(16) double wsm[];
  const int64_t mbp = (max_blocks + 31) & ~int64_t(31);
  double* part = wsm;                          // [kLevels][mbp]
  double* u_in = part + kLevels * mbp;         // [mbp]
  double* u_out = u_in + mbp;                  // [mbp]
  double* ub = u_out + mbp;                    // [2][32][kLevels]: u_l of a block's rows (by block parity)
  uint32_t* ad2 = reinterpret_cast<uint32_t*>(ub + 2 * 32 * kLevels);  // [2][32][33]: diagonal triangles
  uint32_t* ar2 = ad2 + 2 * 32 * 33;           // [2][32][32]: a row block's entries in the columns of the block below
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t unit = blockIdx.x;
  const int bi = static_cast<int>(unit / hq);
  const int32_t len = seq_lens[bi];
  if (len < 1 || len > max_len) {
    if (tid == 0) record_error(err, GUARD_BAD_LEN);
    return;
  }
  const int nb = static_cast<int>((len - 1) / B + 1);
  const int i = nb - 1;
  const uint32_t* A = rows + unit * rows_offset(max_blocks);
  double* wrow = walk_state + unit * max_blocks;
  for (int j = tid; j < nb; j += kWalkThreads) u_in[j] = first_layer ? (j == i ? 1.0 : 0.0) : wrow[j];
  const int mtop = (i / 32) * 32;

  // warp 1 loads into shared memory the entries the chain's next step reads:
  // the triangle of block T in ad[r][.] (row T + r; zeros above the diagonal
  // and past the newest row) and, for T < M, the rows of block M in the
  // columns of block T in ar[r][.], into the buffers of T's parity, which the
  // chain last read a step earlier.
  auto stage = [&](int T, int M) {
    const int c = T + lane;
    uint32_t* ad = ad2 + ((T >> 5) & 1) * 32 * 33;
    uint32_t* ar = ar2 + ((T >> 5) & 1) * 32 * 32;
    uint32_t v[16];  // sixteen rows' entries in flight at once
#pragma unroll
    for (int h = 0; h < 32; h += 16) {
#pragma unroll
      for (int r = 0; r < 16; ++r)
        v[r] = (h + r >= lane && T + h + r <= i) ? __ldg(A + rows_offset(T + h + r) + c) : 0u;
#pragma unroll
      for (int r = 0; r < 16; ++r) ad[(h + r) * 33 + lane] = v[r];
    }
    if (T < M) {
#pragma unroll
      for (int h = 0; h < 32; h += 16) {
#pragma unroll
        for (int r = 0; r < 16; ++r) v[r] = M + h + r <= i ? __ldg(A + rows_offset(M + h + r) + c) : 0u;
#pragma unroll
        for (int r = 0; r < 16; ++r) ar[(h + r) * 32 + lane] = v[r];
      }
    }
  };

  // warp 0: the diagonal triangle of block M (its columns' part complete, its
  // triangle staged in ad)
  auto diag = [&](int M, int L) {
    const int m = M + lane;
    const bool live = m <= i;
    double* ubm = ub + ((M >> 5) & 1) * 32 * kLevels;
    const uint32_t* ad = ad2 + ((M >> 5) & 1) * 32 * 33;
    double uprev = live ? u_in[m] : 0.0;
    for (int l = 0; l < kLevels; ++l) {
      if (l >= L) {  // levels past this sweep's: zeros, so every product that reads them adds 0
        ubm[lane * kLevels + l] = 0.0;
        continue;
      }
      ubm[lane * kLevels + l] = uprev;
      // eight interleaved partial sums (rows r mod 8), added in a fixed order
      double acc[8] = {live ? part[l * mbp + m] : 0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0};
#pragma unroll
      for (int r = 31; r >= 0; --r) {
        const double v = __shfl_sync(0xffffffffu, uprev, r);
        acc[r & 7] = fma(v, from_hi(ad[r * 33 + lane]), acc[r & 7]);
      }
      uprev = ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
    }
    if (live) u_out[m] = uprev;
  };

  // The rows of block M (rows M .. M + 31 up to the newest), pulled into L2 two
  // blocks ahead of their reads by one warp (a bulk prefetch per row), so that
  // the many small row reads of the other warps find them there.
  auto prefetch_block = [&](int M) {
    if (M < 0) return;
    const int m = M + lane;
    if (m <= i) prefetch_l2(A + rows_offset(m), static_cast<uint32_t>(((m + 1 + 3) & ~3) * 4));
  };
  for (int done = 0; done < s_pow; done += kLevels) {
    const int L = min(kLevels, s_pow - done);
    if (warp == 1) {
      prefetch_block(mtop);
      prefetch_block(mtop - 32);
    }
    for (int x = tid; x < kLevels * mbp; x += kWalkThreads) part[x] = 0.0;
    if (warp == 1) {
      stage(mtop, mtop);
      if (mtop > 0) stage(mtop - 32, mtop);
    }
    __syncthreads();
    if (warp == 0) diag(mtop, L);
    __syncthreads();
    for (int M = mtop; M > 0; M -= 32) {
      const int nrows = min(32, i - M + 1);
      const double* ubm = ub + ((M >> 5) & 1) * 32 * kLevels;
      if (warp == 1) {
        // the entries the chain reads at the next block, staged while it works on this one
        prefetch_block(M - 64);
        if (M - 32 > 0) stage(M - 64, M - 32);
      } else if (warp == 0) {
        // block M's rows into the columns of block M - 32, then that block's
        // diagonal; both were staged during the previous step
        const int c = M - 32 + lane;
        const uint32_t* ar = ar2 + (((M - 32) >> 5) & 1) * 32 * 32;
        double acc[2][kLevels];  // rows of even and odd index, added at the end
#pragma unroll
        for (int l = 0; l < kLevels; ++l) acc[0][l] = acc[1][l] = 0.0;
#pragma unroll
        for (int r = 0; r < 32; ++r) {
          const double a = from_hi(ar[r * 32 + lane]);
#pragma unroll
          for (int l = 0; l < kLevels; ++l) acc[r & 1][l] = fma(ubm[r * kLevels + l], a, acc[r & 1][l]);
        }
        for (int l = 0; l < L; ++l) part[l * mbp + c] += acc[0][l] + acc[1][l];
        __syncwarp();
        diag(M - 32, L);
      } else {
        // block M's rows into the columns left of block M - 32 on the fp64 tensor
        // path: per 16 columns, D[column][level] += sum over the block's rows r of
        // A[M + r][column] u_level[M + r], i.e. D (16 x 8) += A^T (16 x 4) U (4 x 8)
        // over the block's 32 rows in 8 products of m16n8k4 (the 8 levels are n).
        // Lane (g, t4) holds A at rows 4 kk + t4, columns g and g + 8 of the chunk.
        const int g = lane >> 2, t4 = lane & 3;
        const int nchunk = (M - 32) / 16;
        const int wk = warp - 2;
        uint32_t cur[8][2], nxt[8][2];
        auto load_chunk = [&](int ch, uint32_t (&dst)[8][2]) {
          const int c0 = 16 * ch;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const int r = 4 * kk + t4;
            const uint32_t* row = A + rows_offset(M + r);
            const bool ok = r < nrows;
            dst[kk][0] = ok ? __ldg(row + c0 + g) : 0u;
            dst[kk][1] = ok ? __ldg(row + c0 + g + 8) : 0u;
          }
        };
        if (wk < nchunk) load_chunk(wk, cur);
        for (int ch = wk; ch < nchunk; ch += kWalkWarps - 2) {
          const int nc = ch + kWalkWarps - 2;
          if (nc < nchunk) load_chunk(nc, nxt);
          double acc[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            dmma_16x8x4(acc, from_hi(cur[kk][0]), from_hi(cur[kk][1]), ubm[(4 * kk + t4) * kLevels + g]);
          // acc: D[g][2 t4], D[g][2 t4 + 1], D[g + 8][2 t4], D[g + 8][2 t4 + 1]
          const int c0 = 16 * ch;
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int l = 2 * t4 + e;
            if (l < L) {
              part[l * mbp + c0 + g] += acc[e];
              part[l * mbp + c0 + g + 8] += acc[2 + e];
            }
          }
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            cur[kk][0] = nxt[kk][0];
            cur[kk][1] = nxt[kk][1];
          }
        }
      }
      __syncthreads();
    }
    for (int j = tid; j < nb; j += kWalkThreads) u_in[j] = u_out[j];
    __syncthreads();
  }
  for (int j = tid; j < nb; j += kWalkThreads) wrow[j] = u_in[j];
}

size_t walk_smem_bytes(int64_t max_blocks) {
  const size_t mbp = static_cast<size_t>((max_blocks + 31) & ~int64_t(31));
  return ((kLevels + 2) * mbp + 2 * 32 * kLevels) * sizeof(double) + 2 * (32 * 33 + 32 * 32) * sizeof(uint32_t);
}

// Step part 3: per head the top-tau of its row (or the group's summed rows for
// a shared choice), then the union over the group with its head mask.
constexpr int kSelThreads = 512;
constexpr int kSelWarps = kSelThreads / 32;

__global__ void __launch_bounds__(kSelThreads) exact_select_kernel(
    const double* __restrict__ walk_state, int32_t hq, int32_t hkv, int64_t max_len, int64_t max_blocks,
    const int32_t* __restrict__ seq_lens, int32_t B, int32_t num, int32_t den, int shared,
    int32_t* __restrict__ head_sel, int32_t* __restrict__ head_cnt, int32_t* __restrict__ sel,
    uint8_t* __restrict__ sel_mask, int32_t* __restrict__ sel_cnt, int32_t* err) {
  grid_dependency_wait();
  allow_dependents();
  const int group = hq / hkv;
  extern __shared__ __align__(16) uint8_t ssm[];
  uint64_t* keys = reinterpret_cast<uint64_t*>(ssm);             // [group][max_blocks]
  uint32_t* mark = reinterpret_cast<uint32_t*>(keys + (int64_t)group * max_blocks);  // [max_blocks]
  int* hist = reinterpret_cast<int*>(mark + ((max_blocks + 3) & ~int64_t(3)));        // [group][256]
  int* ctl = hist + group * 256;                                  // [group][4]
  int* wsum = ctl + group * 4;                                    // [kSelWarps]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t unit = blockIdx.x;
  const int bi = static_cast<int>(unit / hkv), g = static_cast<int>(unit % hkv);
  const int32_t len = seq_lens[bi];
  if (len < 1 || len > max_len) {
    if (tid == 0) record_error(err, GUARD_BAD_LEN);
    return;
  }
  const int nb = static_cast<int>((len - 1) / B + 1);
  const int i = nb - 1;
  const int64_t h0 = (int64_t)bi * hq + (int64_t)g * group;
  for (int j = tid; j < nb; j += kSelThreads) mark[j] = 0u;
  if (!shared) {
    for (int x = tid; x < group * nb; x += kSelThreads) {
      const int r = x / nb, j = x % nb;
      keys[(int64_t)r * max_blocks + j] = order_key(walk_state[(h0 + r) * max_blocks + j]);
    }
  } else {
    for (int j = tid; j < nb; j += kSelThreads) {
      double sm = walk_state[h0 * max_blocks + j];
      for (int q = 1; q < group; ++q) sm += walk_state[(h0 + q) * max_blocks + j];
      keys[j] = order_key(sm);
    }
  }
  __syncthreads();
  const int tau = tau_of_row(i, num, den);
  if (!shared) {
    const int wph = kSelWarps / group;  // >= 1 since group <= 8
    const int r = warp / wph;
    if (r < group) {
      const int t = tid - r * wph * 32, nthr = wph * 32, bar_id = 1 + r;
      group_top_tau(keys + (int64_t)r * max_blocks, nb, tau, hist + r * 256, ctl + r * 4, t, nthr, bar_id,
                    head_sel + (h0 + r) * max_blocks, mark, 1u << r, err);
      if (t == 0) head_cnt[h0 + r] = tau;
    }
    __syncthreads();
  } else {
    int32_t* sel0 = head_sel + h0 * max_blocks;
    group_top_tau(keys, nb, tau, hist, ctl, tid, kSelThreads, 1, sel0, mark, (1u << group) - 1u, err);
    __syncthreads();
    for (int q = 1; q < group; ++q)
      for (int x = tid; x < tau; x += kSelThreads) sel0[(int64_t)q * max_blocks + x] = sel0[x];
    if (tid < group) head_cnt[h0 + tid] = tau;
    __syncthreads();
  }
  // ordered compaction of the union
  int base = 0;
  for (int j0 = 0; j0 < nb; j0 += kSelThreads) {
    const int j = j0 + tid;
    const uint32_t mk = (j < nb) ? mark[j] : 0u;
    const unsigned bal = __ballot_sync(0xffffffffu, mk != 0u);
    if (lane == 0) wsum[warp] = __popc(bal);
    __syncthreads();
    int off = base;
    for (int w = 0; w < warp; ++w) off += wsum[w];
    int tot = 0;
    for (int w = 0; w < kSelWarps; ++w) tot += wsum[w];
    if (mk != 0u) {
      const int p = off + __popc(bal & lanemask_lt());
      sel[unit * max_blocks + p] = static_cast<int32_t>(j);
      sel_mask[unit * max_blocks + p] = static_cast<uint8_t>(mk);
    }
    base += tot;
    __syncthreads();
  }
  if (tid == 0) sel_cnt[unit] = base;
}

size_t select_smem_bytes(int64_t max_blocks, int group) {
  return static_cast<size_t>(group) * max_blocks * 8 + ((max_blocks + 3) & ~int64_t(3)) * 4 +
         static_cast<size_t>(group) * 256 * 4 + static_cast<size_t>(group) * 4 * 4 + kSelWarps * 4;
}

cudaError_t launch_walk(const uint32_t* rows, int64_t max_len, int64_t mb, int32_t batch, int32_t hq,
                        const int32_t* seq_lens, int32_t B, int first_layer, int32_t s_pow, double* walk_state,
                        int32_t* err, cudaStream_t st) {
  const size_t smem = walk_smem_bytes(mb);
  const cudaError_t e = cudaFuncSetAttribute(exact_walk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_k(exact_walk_kernel, static_cast<unsigned>((int64_t)batch * hq), kWalkThreads, smem, st, rows,
                  max_len, mb, seq_lens, B, hq, first_layer, s_pow, walk_state, err);
}

}  // namespace

int64_t exact_rows_entries(int64_t max_blocks) { return rows_offset(max_blocks); }

bool exact_wide_supported(const sws_config& c, int64_t max_blocks, int32_t group) {
  return c.sketch_dim <= kMaxK && group >= 1 && group <= 8 && max_blocks <= 2560 &&
         walk_smem_bytes(max_blocks) <= (227u << 10) &&
         select_smem_bytes(max_blocks, group) <= (227u << 10) &&
         rows_smem_bytes(c.sketch_dim, group, 32) <= (200u << 10);
}

cudaError_t launch_exact_rows_init(const sws_handle* h, const double* q_sketch, const double* k_sketch, int32_t batch,
                                   int32_t hq, int32_t hkv, int64_t max_len, const int32_t* seq_lens, uint32_t* rows,
                                   cudaStream_t st) {
  const sws_config& c = h->cfg;
  const int64_t mb = ceil_div64(max_len, c.block_size);
  const size_t smem = rows_smem_bytes(c.sketch_dim, hq / hkv, 32);
  cudaError_t e = cudaFuncSetAttribute(exact_rows_init_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(static_cast<unsigned>((int64_t)batch * hkv), static_cast<unsigned>(ceil_div64(mb, 32)));
  e = launch_k(exact_rows_init_kernel, grid, kRowThreads, smem, st, q_sketch, k_sketch, hq, hkv, max_len, mb, seq_lens,
               c.block_size, c.sketch_dim, rows, h->err);
  if (e != cudaSuccess) return e;
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_decode_exact_wide(const sws_handle* h, const __nv_bfloat16* q_tok, const __nv_bfloat16* k_tok,
                                     const __nv_bfloat16* v_tok, int32_t batch, int32_t hq, int32_t hkv,
                                     int64_t max_len, const int32_t* seq_lens, __nv_bfloat16* k_cache,
                                     __nv_bfloat16* v_cache, double* k_psum, double* k_sketch, double* q_psum,
                                     double* q_sketch, uint32_t* rows, int first_layer, double* walk_state,
                                     int32_t* head_sel, int32_t* head_cnt, int32_t* sel, uint8_t* sel_mask,
                                     int32_t* sel_cnt, cudaStream_t st) {
  const sws_config& c = h->cfg;
  const int64_t mb = ceil_div64(max_len, c.block_size);
  const int group = hq / hkv;
  const unsigned units_kv = static_cast<unsigned>((int64_t)batch * hkv);
  // 1. append and the newest rows
  {
    const int D = c.head_dim;
    const size_t smem = (rows_smem_bytes(c.sketch_dim, group, 1) + 15) / 16 * 16 + (size_t)(1 + group) * D * 8;
    auto kern = D == 128 ? exact_append_rows_kernel<128> : exact_append_rows_kernel<64>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = launch_k(kern, units_kv, kRowThreads, smem, st, q_tok, k_tok, v_tok, hq, hkv, max_len, mb, seq_lens, k_cache,
                 v_cache, k_psum, k_sketch, q_psum, q_sketch, h->hdt, c.sketch_dim, c.block_size, rows, h->err);
    if (e != cudaSuccess) return e;
  }
  // 2. the walk row of every head
  {
    const cudaError_t e = launch_walk(rows, max_len, mb, batch, hq, seq_lens, c.block_size, first_layer, c.walk_power,
                                      walk_state, h->err, st);
    if (e != cudaSuccess) return e;
  }
  // 3. selection and union
  {
    const size_t smem = select_smem_bytes(mb, group);
    cudaError_t e = cudaFuncSetAttribute(exact_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = launch_k(exact_select_kernel, units_kv, kSelThreads, smem, st, walk_state, hq, hkv, max_len, mb, seq_lens,
                 c.block_size, c.density_num, c.density_den, (c.select_group > 1 && group > 1) ? 1 : 0, head_sel,
                 head_cnt, sel, sel_mask, sel_cnt, h->err);
    if (e != cudaSuccess) return e;
  }
  note_launches(3);
  return cudaGetLastError();
}

}  // namespace sws
