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
// One CTA of 1024 threads per (sequence, KV head), as in decode_select_kernel:
//  1. append the token's K/V, update the key and query block sums and the last
//     block's k~ and (per query head of the group) q~;
//  2. stage k~ of every block in shared memory (fp32, rows padded to k + 1);
//  3. per query head: A as fp32 in shared memory (one warp per row: the scores
//     on fp32 FMA, the row maximum, exponentials, the row sum in fp64), then
//     the s products u <- u A in fp64, each column's sum cut into slices of
//     rows that are added in a fixed order;
//  4. per head (or per group, for group-shared selection) the top-tau of u,
//     then the union over the group with its head mask.
#include <algorithm>

#include "select.cuh"
#include "sws_common.cuh"

namespace sws {
namespace {

constexpr int kExThreads = 1024;
constexpr int kExWarps = kExThreads / 32;
constexpr int kExMaxK = 32;     // sketch dims held in registers per lane
constexpr int kExSlices = 4;    // row slices of one product's column sums

__host__ __device__ constexpr int64_t tri_count(int64_t nb) { return nb * (nb + 1) / 2; }

// Shared-memory carve-up for max_blocks blocks; every part 16-byte aligned.
struct ExactSmem {
  int64_t a, ks, u, part, keys, mark, mean, qrow, hist, ctl, wsum, total;
  __host__ __device__ ExactSmem(int64_t mb, int group, int k, int D) {
    auto up = [](int64_t x) { return (x + 15) & ~int64_t(15); };
    a = 0;                                                  // float [tri(mb)]
    ks = up(a + tri_count(mb) * 4);                         // float [mb][k + 1]
    u = up(ks + mb * (k + 1) * 4);                          // double [2][mb]
    part = up(u + 2 * mb * 8);                              // double [kExSlices][mb]
    keys = up(part + kExSlices * mb * 8);                   // uint64 [group][mb] (u rows for a shared choice)
    mark = up(keys + (int64_t)group * mb * 8);              // uint32 [mb]
    mean = up(mark + mb * 4);                               // double [D]
    qrow = up(mean + D * 8);                                // double [group][D]
    hist = up(qrow + (int64_t)group * D * 8);               // int [group][256]
    ctl = up(hist + (int64_t)group * 256 * 4);              // int [group][4]
    wsum = up(ctl + (int64_t)group * 4 * 4);                // int [kExWarps + 1]
    total = up(wsum + (kExWarps + 1) * 4);
  }
};

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
  float* A = reinterpret_cast<float*>(smem + L.a);
  float* ks = reinterpret_cast<float*>(smem + L.ks);
  double* ubuf = reinterpret_cast<double*>(smem + L.u);
  double* part = reinterpret_cast<double*>(smem + L.part);
  uint64_t* keys = reinterpret_cast<uint64_t*>(smem + L.keys);
  uint32_t* mark = reinterpret_cast<uint32_t*>(smem + L.mark);
  double* mean = reinterpret_cast<double*>(smem + L.mean);
  double* qrow = reinterpret_cast<double*>(smem + L.qrow);
  int* hist = reinterpret_cast<int*>(smem + L.hist);
  int* ctl = reinterpret_cast<int*>(smem + L.ctl);
  int* wsum = reinterpret_cast<int*>(smem + L.wsum);
  const int ksp = k + 1;  // padded k~ row (floats): lanes on consecutive rows hit consecutive banks

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

  // 2. k~ of every block, fp32, padded rows
  for (int x = tid; x < nb * k; x += kExThreads) ks[(x / k) * ksp + x % k] = static_cast<float>(ksk[x]);
  __syncthreads();

  const float inv_sqrt_k = static_cast<float>(1.0 / sqrt(static_cast<double>(k)));
  const int ntiles = (nb + 31) / 32;
  for (int r = 0; r < group; ++r) {
    const int64_t h = (int64_t)g * group + r;
    const double* qsk = q_sketch + ((int64_t)bi * hq + h) * max_blocks * k;
    // 3a. A = row softmax of S over j <= m, fp32, row m at offset m (m + 1) / 2
    for (int m = warp; m < nb; m += kExWarps) {
      float qv[kExMaxK];
#pragma unroll
      for (int c = 0; c < kExMaxK; ++c) qv[c] = c < k ? static_cast<float>(qsk[(int64_t)m * k + c]) : 0.f;
      float* arow = A + tri_count(m);
      float mx = -INFINITY;
      for (int j = lane; j <= m; j += 32) {
        const float* kr = ks + j * ksp;
        float sdot = 0.f;
#pragma unroll
        for (int c = 0; c < kExMaxK; ++c)
          if (c < k) sdot = fmaf(qv[c], kr[c], sdot);
        sdot *= inv_sqrt_k;
        arow[j] = sdot;
        mx = fmaxf(mx, sdot);
      }
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
      const float inv = static_cast<float>(1.0 / se);
      for (int j = lane; j <= m; j += 32) arow[j] *= inv;
    }
    // 3b. u: e_i on the first layer, else the previous layer's row
    double* u0 = ubuf;
    double* u1 = ubuf + max_blocks;
    double* wrow = walk_state + ((int64_t)bi * hq + h) * max_blocks;
    for (int j = tid; j < nb; j += kExThreads) u0[j] = first_layer ? (j == i ? 1.0 : 0.0) : wrow[j];
    __syncthreads();
    // 3c. s products u <- u A: column j sums u_m A_mj over m >= j; warp w
    //     takes column tile w % ntiles and the rows of slice w / ntiles
    const int fit = kExWarps / ntiles;  // >= 1 since nb <= kExThreads
    const int slices = fit < kExSlices ? (fit < 1 ? 1 : fit) : kExSlices;
    const int rows_per = (nb + slices - 1) / slices;
    for (int p = 0; p < s_pow; ++p) {
      if (warp < ntiles * slices) {
        const int j = (warp % ntiles) * 32 + lane;
        const int sl = warp / ntiles;
        const int m0 = std::max(j, sl * rows_per), m1 = std::min(nb, (sl + 1) * rows_per);
        double acc = 0.0;
        if (j < nb)
          for (int m = m0; m < m1; ++m) acc = fma(u0[m], static_cast<double>(A[tri_count(m) + j]), acc);
        if (j < nb) part[sl * max_blocks + j] = acc;
      }
      __syncthreads();
      for (int j = tid; j < nb; j += kExThreads) {
        double acc = part[j];
        for (int sl = 1; sl < slices; ++sl) acc += part[sl * max_blocks + j];
        u1[j] = acc;
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
  return cfg.sketch_dim <= kExMaxK && max_blocks <= kExThreads && group >= 1 && group <= 8 &&
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
