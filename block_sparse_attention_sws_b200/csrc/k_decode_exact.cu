// Exact decode walk: the selection of the new token's query block is the last
// row of the prefill recurrence of "Scout Before You Attend" §4, computed on
// the sequence as it stands (prompt plus the tokens decoded so far).
//
// For query block i = nb - 1 (the block of the new token) and layer l:
//   R^l[i] = R^{l-1}[i] (A^l)^s,  R^0[i] = e_i (A^0)^s,
// so the row is carried across the layers of one step as a vector u and
// advanced by s products u <- u A^l, where A^l is the row softmax (j <= m) of
// the sketched scores S_mj = q~_m . k~_j / sqrt(k) of this layer. The query
// sketches q~_m of the earlier blocks are cached (from the prefill and from
// earlier steps); the last block's q~ is the projection of the mean of its
// queries so far, like its key sketch. The row costs O(s b^2) per head and
// layer, against O(b) for the log-domain walk of sws_decode_step.
//
// One CTA of 512 threads per (sequence, KV head), as in decode_select_kernel:
//  1. append the token's K/V, update the key and query block sums and the last
//     block's k~ and (per query head of the group) q~;
//  2. stage k~ of every block in shared memory (fp32); per query head: the
//     scores S on fp32 FMA (32-column tiles with k~ in registers and q~
//     broadcast from shared memory) into a triangle of 4-byte slots; per row
//     the maximum, exponentials, the row sum and the normalisation in fp64,
//     each entry of A stored back as the rounded high word of its fp64 value;
//     then the s products u <- u A in fp64, balanced over the triangle by
//     pairing column j with column nb - 1 - j;
//  3. per head (or per group, for group-shared selection) the top-tau of u,
//     then the union over the group with its head mask.
//
// Measured at a 16K-token prompt (257 blocks, group of 4): about 38 us of
// scores and softmax and 33 us of products per head and layer; the products
// issue about 500 instructions a lane at ~30% issue efficiency with four
// warps per sub-partition, which the 224 KB of shared memory allows.
#include <algorithm>

#include "select.cuh"
#include "sws_common.cuh"

namespace sws {
namespace {

constexpr int kExThreads = 512;  // 16 warps: up to 128 registers a thread
constexpr int kExWarps = kExThreads / 32;
constexpr int kExMaxK = 32;     // sketch dims held in registers per lane

__host__ __device__ constexpr int64_t tri_count(int64_t nb) { return nb * (nb + 1) / 2; }
__device__ __forceinline__ int tri32(int m) { return (m * (m + 1)) >> 1; }  // m < 2^15

// The normalised block attention is kept as the high 32 bits of its fp64 value
// (sign, 11-bit exponent, 20-bit mantissa, rounded to nearest): the same 4
// bytes as an fp32, the fp64 exponent range, a relative precision of 2^-21,
// and an fp64 operand for the products from a register move, no conversion.
__device__ __forceinline__ uint32_t to_hi20(double x) {
  const uint64_t b = static_cast<uint64_t>(__double_as_longlong(x)) + 0x80000000ull;
  return static_cast<uint32_t>(b >> 32);
}
__device__ __forceinline__ double from_hi20(uint32_t h) { return __hiloint2double(static_cast<int>(h), 0); }

// Shared-memory carve-up for max_blocks blocks; every part 16-byte aligned.
struct ExactSmem {
  int64_t a, qs, ks, u, part, keys, mark, mean, qrow, hist, ctl, wsum, total;
  __host__ __device__ ExactSmem(int64_t mb, int group, int k, int D) {
    auto up = [](int64_t x) { return (x + 15) & ~int64_t(15); };
    a = 0;                                                  // float [tri(mb)]
    qs = up(a + tri_count(mb) * 4);                         // float [mb][k]: one head's q~
    ks = up(qs + mb * k * 4);                               // float [mb][k + 1]: the KV head's k~
    u = up(ks + mb * (k + 1) * 4);                          // double [2][mb]
    part = up(u + 2 * mb * 8);                              // double [mb]
    keys = up(part + mb * 8);                               // uint64 [group][mb] (u rows for a shared choice)
    mark = up(keys + (int64_t)group * mb * 8);              // uint32 [mb]
    mean = up(mark + mb * 4);                               // double [D]
    qrow = up(mean + D * 8);                                // double [group][D]
    hist = up(qrow + (int64_t)group * D * 8);               // int [group][256]
    ctl = up(hist + (int64_t)group * 256 * 4);              // int [group][4]
    wsum = up(ctl + (int64_t)group * 4 * 4);                // int [kExWarps + 1]
    total = up(wsum + (kExWarps + 1) * 4);
  }
};

// sum over m = m0, m0 + step, ... < nb of u[m] A[m][j], in four interleaved
// chains added in a fixed order (fp64; A from the triangle of high words)
__device__ __forceinline__ double column_dot(const double* u, const uint32_t* A, int m0, int step, int nb, int j) {
  double c0 = 0.0, c1 = 0.0, c2 = 0.0, c3 = 0.0;
  int m = m0;
  for (; m + 3 * step < nb; m += 4 * step) {
    c0 = fma(u[m], from_hi20(A[tri32(m) + j]), c0);
    c1 = fma(u[m + step], from_hi20(A[tri32(m + step) + j]), c1);
    c2 = fma(u[m + 2 * step], from_hi20(A[tri32(m + 2 * step) + j]), c2);
    c3 = fma(u[m + 3 * step], from_hi20(A[tri32(m + 3 * step) + j]), c3);
  }
  for (; m < nb; m += step) c0 = fma(u[m], from_hi20(A[tri32(m) + j]), c0);
  return (c0 + c1) + (c2 + c3);
}

template <int D>
__global__ void __launch_bounds__(kExThreads) decode_exact_kernel(
    const __nv_bfloat16* __restrict__ q_tok, const __nv_bfloat16* __restrict__ k_tok,
    const __nv_bfloat16* __restrict__ v_tok, int32_t hq, int32_t hkv, int64_t max_len, int64_t max_blocks,
    const int32_t* __restrict__ seq_lens, __nv_bfloat16* __restrict__ k_cache, __nv_bfloat16* __restrict__ v_cache,
    double* __restrict__ k_psum, double* __restrict__ k_sketch, double* __restrict__ q_psum,
    double* __restrict__ q_sketch, int first_layer, double* __restrict__ walk_state, int32_t* __restrict__ head_sel,
    int32_t* __restrict__ head_cnt, int32_t* __restrict__ sel, uint8_t* __restrict__ sel_mask,
    int32_t* __restrict__ sel_cnt, const double* __restrict__ hdt, int32_t k, int32_t B, int32_t s_pow, int32_t num,
    int32_t den, int shared, int32_t* err) {
  grid_dependency_wait();
  allow_dependents();
  const int group = hq / hkv;
  extern __shared__ __align__(16) uint8_t smem[];
  const ExactSmem L(max_blocks, group, k, D);
  float* A = reinterpret_cast<float*>(smem + L.a);  // scores, then (as Ah) the attention's high words
  const uint32_t* Ah = reinterpret_cast<const uint32_t*>(smem + L.a);
  float* qs = reinterpret_cast<float*>(smem + L.qs);
  float* ks = reinterpret_cast<float*>(smem + L.ks);
  const int ksp = k + 1;  // padded k~ rows: lanes on consecutive rows read consecutive banks
  double* ubuf = reinterpret_cast<double*>(smem + L.u);
  double* part = reinterpret_cast<double*>(smem + L.part);
  uint64_t* keys = reinterpret_cast<uint64_t*>(smem + L.keys);
  uint32_t* mark = reinterpret_cast<uint32_t*>(smem + L.mark);
  double* mean = reinterpret_cast<double*>(smem + L.mean);
  double* qrow = reinterpret_cast<double*>(smem + L.qrow);
  int* hist = reinterpret_cast<int*>(smem + L.hist);
  int* ctl = reinterpret_cast<int*>(smem + L.ctl);
  int* wsum = reinterpret_cast<int*>(smem + L.wsum);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t unit = blockIdx.x;
  const int bi = static_cast<int>(unit / hkv), g = static_cast<int>(unit % hkv);
  const int32_t len = seq_lens[bi];
  if (len < 1 || len > max_len) {
    if (tid == 0) record_error(err, GUARD_BAD_LEN);
    return;
  }
  const int64_t pos = len - 1;
  const int64_t blk = pos / B;
  const int cnt = static_cast<int>(pos % B) + 1;
  const int nb = static_cast<int>(blk + 1);
  const int i = nb - 1;
  for (int j = tid; j < nb; j += kExThreads) mark[j] = 0u;

  // 1. append the token; the key and query sums of the last block and their means
  if (tid < D) {
    const __nv_bfloat16 kt = k_tok[unit * D + tid];
    k_cache[(unit * max_len + pos) * D + tid] = kt;
    v_cache[(unit * max_len + pos) * D + tid] = v_tok[unit * D + tid];
    double ps = (cnt == 1) ? 0.0 : k_psum[unit * D + tid];
    ps += static_cast<double>(__bfloat162float(kt));
    k_psum[unit * D + tid] = ps;
    mean[tid] = ps / cnt;
  }
  for (int x = tid; x < group * D; x += kExThreads) {
    const int64_t h = (int64_t)g * group + x / D;
    const int c = x % D;
    const int64_t qi = ((int64_t)bi * hq + h) * D + c;
    double ps = (cnt == 1) ? 0.0 : q_psum[qi];
    ps += static_cast<double>(__bfloat162float(q_tok[qi]));
    q_psum[qi] = ps;
    qrow[x] = ps / cnt;
  }
  __syncthreads();
  // the last block's k~ and, per query head, its q~; one warp per output
  double* ksk = k_sketch + unit * max_blocks * k;
  for (int o = warp; o < (group + 1) * k; o += kExWarps) {
    const int r = o / k, c = o % k;  // r == group: the key block
    const double v = warp_dot_hdt<D>(r == group ? mean : qrow + r * D, hdt + (size_t)c * D, lane);
    if (lane == 0) {
      if (r == group) ksk[(int64_t)i * k + c] = v;
      else q_sketch[(((int64_t)bi * hq + (int64_t)g * group + r) * max_blocks + i) * k + c] = v;
    }
  }
  __syncthreads();  // the CTA's global writes above are visible to it after the barrier
  // 2. k~ of every block, fp32, in shared memory (coalesced reads; shared by the group's heads)
  for (int x = tid; x < nb * k; x += kExThreads) ks[(x / k) * ksp + x % k] = static_cast<float>(ksk[x]);

  const float inv_sqrt_k = static_cast<float>(1.0 / sqrt(static_cast<double>(k)));
  for (int r = 0; r < group; ++r) {
    const int64_t h = (int64_t)g * group + r;
    const double* qsk = q_sketch + ((int64_t)bi * hq + h) * max_blocks * k;
    // 3a. the scores S_mj, fp32, into the triangle (row m at offset m (m + 1) / 2).
    //     A warp works down one 32-column tile at a time with its lane's k~_j
    //     in registers, reading each row's q~ as 16-byte broadcasts from shared
    //     memory: four FMAs per shared load. The (tile, row) items, rows
    //     m >= 32 J of tile J, are dealt to the warps in order.
    for (int x = tid; x < nb * k; x += kExThreads) qs[x] = static_cast<float>(qsk[x]);
    __syncthreads();
    {
      const int ntiles = (nb + 31) / 32;
      int tile = -1, tile_first = 0;  // the tile of the registers and its first item index
      float kreg[kExMaxK];
      int jt = 0, start = 0;          // walking the tiles: tile jt covers items [start, start + nb - 32 jt)
      for (int x = warp; ; x += kExWarps) {
        while (jt < ntiles && x >= start + (nb - 32 * jt)) {
          start += nb - 32 * jt;
          ++jt;
        }
        if (jt >= ntiles) break;
        if (jt != tile) {
          tile = jt;
          tile_first = start;
          const int j = 32 * tile + lane;
#pragma unroll
          for (int c = 0; c < kExMaxK; ++c) kreg[c] = (c < k && j < nb) ? ks[j * ksp + c] : 0.f;
        }
        const int m = 32 * tile + (x - tile_first);
        const int j = 32 * tile + lane;
        const float4* q4 = reinterpret_cast<const float4*>(qs + m * k);
        float sdot = 0.f;
#pragma unroll
        for (int c4 = 0; c4 < kExMaxK / 4; ++c4) {
          if (4 * c4 < k) {
            const float4 qv = q4[c4];
            sdot = fmaf(qv.x, kreg[4 * c4], sdot);
            sdot = fmaf(qv.y, kreg[4 * c4 + 1], sdot);
            sdot = fmaf(qv.z, kreg[4 * c4 + 2], sdot);
            sdot = fmaf(qv.w, kreg[4 * c4 + 3], sdot);
          }
        }
        if (j <= m) A[tri32(m) + j] = sdot * inv_sqrt_k;
      }
    }
    __syncthreads();
    // 3a'. row softmax over j <= m, one warp per row: maximum, exponentials
    //      (the sum in fp64), normalisation in fp64, stored as high words
    for (int m = warp; m < nb; m += kExWarps) {
      float* arow = A + tri32(m);
      float mx = -INFINITY;
      for (int j = lane; j <= m; j += 32) mx = fmaxf(mx, arow[j]);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      double se = 0.0;
      for (int j = lane; j <= m; j += 32) {
        const float e = expf(arow[j] - mx);
        arow[j] = e;
        se += static_cast<double>(e);
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) se += __shfl_xor_sync(0xffffffffu, se, off);
      const double inv = 1.0 / se;
      uint32_t* hrow = reinterpret_cast<uint32_t*>(arow);
      for (int j = lane; j <= m; j += 32) hrow[j] = to_hi20(static_cast<double>(arow[j]) * inv);
    }
    // 3b. u: e_i on the first layer, else the previous layer's row
    double* u0 = ubuf;
    double* u1 = ubuf + max_blocks;
    double* wrow = walk_state + ((int64_t)bi * hq + h) * max_blocks;
    for (int j = tid; j < nb; j += kExThreads) u0[j] = first_layer ? (j == i ? 1.0 : 0.0) : wrow[j];
    __syncthreads();
    // 3c. s products u <- u A. Column j sums u_m A_mj over m >= j; columns j
    //     and nb - 1 - j together have nb + 1 terms, so a group of 4 lanes
    //     takes such a pair (128 pairs at a time), its lanes striding over the
    //     rows of both columns in eight chains, and adds its lanes with a fixed
    //     shuffle tree (the same order on every run).
    const int npairs = (nb + 1) / 2;
    for (int p = 0; p < s_pow; ++p) {
      for (int base = warp * 8; base < npairs; base += kExThreads / 4) {  // warp-uniform trip count
        const int pr = base + (lane >> 2), sub = lane & 3;
        const int ja = pr, jb = nb - 1 - pr;
        double acc_a = 0.0, acc_b = 0.0;
        if (pr < npairs) {
          acc_a = column_dot(u0, Ah, ja + sub, 4, nb, ja);
          if (jb != ja) acc_b = column_dot(u0, Ah, jb + sub, 4, nb, jb);
        }
#pragma unroll
        for (int off = 1; off < 4; off <<= 1) {
          acc_a += __shfl_xor_sync(0xffffffffu, acc_a, off);
          acc_b += __shfl_xor_sync(0xffffffffu, acc_b, off);
        }
        if (pr < npairs && sub == 0) {
          u1[ja] = acc_a;
          if (jb != ja) u1[jb] = acc_b;
        }
      }
      __syncthreads();
      double* t = u0;
      u0 = u1;
      u1 = t;
    }
    // 3d. the new walk row; its keys (or, for a shared choice, the row itself)
    double* urow = reinterpret_cast<double*>(keys + r * max_blocks);
    for (int j = tid; j < nb; j += kExThreads) {
      wrow[j] = u0[j];
      if (shared) urow[j] = u0[j];
      else keys[r * max_blocks + j] = order_key(u0[j]);
    }
    __syncthreads();  // A and u are rewritten for the next head
  }

  // 4. top-tau per head (its share of the warps), or one choice for the group
  const int tau = tau_of_row(i, num, den);
  if (!shared) {
    const int wph = kExWarps / group;  // >= 1 since group <= 8
    const int r = warp / wph;
    if (r < group) {
      const int t = tid - r * wph * 32, nthr = wph * 32, bar_id = 1 + r;
      const int64_t h = (int64_t)g * group + r;
      group_top_tau(keys + r * max_blocks, nb, tau, hist + r * 256, ctl + r * 4, t, nthr, bar_id,
                    head_sel + ((int64_t)bi * hq + h) * max_blocks, mark, 1u << r, err);
      if (t == 0) head_cnt[(int64_t)bi * hq + h] = tau;
    }
    __syncthreads();
  } else {
    // the top-tau of the sum of the group's rows (added in head order)
    const double* ur = reinterpret_cast<const double*>(keys);
    for (int j = tid; j < nb; j += kExThreads) {
      double sm = ur[j];
      for (int q = 1; q < group; ++q) sm += ur[q * max_blocks + j];
      part[j] = sm;
    }
    __syncthreads();
    for (int j = tid; j < nb; j += kExThreads) keys[j] = order_key(part[j]);
    __syncthreads();
    int32_t* sel0 = head_sel + ((int64_t)bi * hq + (int64_t)g * group) * max_blocks;
    group_top_tau(keys, nb, tau, hist, ctl, tid, kExThreads, 1, sel0, mark, (1u << group) - 1u, err);
    __syncthreads();
    for (int q = 1; q < group; ++q)
      for (int x = tid; x < tau; x += kExThreads) sel0[(int64_t)q * max_blocks + x] = sel0[x];
    if (tid < group) head_cnt[(int64_t)bi * hq + g * group + tid] = tau;
    __syncthreads();
  }

  // 5. ordered compaction of the union
  int base = 0;
  for (int j0 = 0; j0 < nb; j0 += kExThreads) {
    const int j = j0 + tid;
    const uint32_t mk = (j < nb) ? mark[j] : 0u;
    const unsigned bal = __ballot_sync(0xffffffffu, mk != 0u);
    if (lane == 0) wsum[warp] = __popc(bal);
    __syncthreads();
    int off = base;
    for (int w = 0; w < warp; ++w) off += wsum[w];
    int tot = 0;
    for (int w = 0; w < kExWarps; ++w) tot += wsum[w];
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

}  // namespace

size_t decode_exact_smem_bytes(const sws_config& cfg, int64_t max_blocks, int32_t group) {
  return static_cast<size_t>(ExactSmem(max_blocks, group, cfg.sketch_dim, cfg.head_dim).total);
}

bool decode_exact_supported(const sws_config& cfg, int64_t max_blocks, int32_t group) {
  return cfg.sketch_dim <= kExMaxK && cfg.sketch_dim % 4 == 0 && max_blocks <= kExThreads && group >= 1 &&
         group <= 8 &&
         decode_exact_smem_bytes(cfg, max_blocks, group) <= (227u << 10);
}

cudaError_t launch_decode_exact(const sws_handle* h, const __nv_bfloat16* q_tok, const __nv_bfloat16* k_tok,
                                const __nv_bfloat16* v_tok, int32_t batch, int32_t hq, int32_t hkv, int64_t max_len,
                                const int32_t* seq_lens, __nv_bfloat16* k_cache, __nv_bfloat16* v_cache,
                                double* k_psum, double* k_sketch, double* q_psum, double* q_sketch, int first_layer,
                                double* walk_state, int32_t* head_sel, int32_t* head_cnt, int32_t* sel,
                                uint8_t* sel_mask, int32_t* sel_cnt, cudaStream_t st) {
  const sws_config& c = h->cfg;
  const int64_t mb = ceil_div64(max_len, c.block_size);
  const size_t smem = decode_exact_smem_bytes(c, mb, hq / hkv);
  auto kern = c.head_dim == 128 ? decode_exact_kernel<128> : decode_exact_kernel<64>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  {
    const cudaError_t le = launch_k(kern, static_cast<unsigned>((int64_t)batch * hkv), kExThreads, smem, st, q_tok,
                                    k_tok, v_tok, hq, hkv, max_len, mb, seq_lens, k_cache, v_cache, k_psum, k_sketch,
                                    q_psum, q_sketch, first_layer, walk_state, head_sel, head_cnt, sel, sel_mask,
                                    sel_cnt, h->hdt, c.sketch_dim, c.block_size, c.walk_power, c.density_num,
                                    c.density_den, (c.select_group > 1 && hq / hkv > 1) ? 1 : 0, h->err);
    if (le != cudaSuccess) return le;
  }
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace sws
