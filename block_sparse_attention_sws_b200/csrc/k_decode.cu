// Decode-side kernels.
//
// "Scout Before You Attend" §5: every decode step chooses the KV-cache blocks
// for its one new query token with the same sketch-and-walk score, then runs
// exact attention over them (memory-bound: the cost is reading K and V).
//
// Per layer and step:
//   decode_select_kernel (one CTA per (sequence, KV head)):
//     1. appends the token's K/V to the cache, adds K to the running sum of the
//        last block and refreshes that block's sketch k~ = mean * H_d;
//     2. q~ = q H_d for the query heads of the GQA group and z_j = q~ . k~_j /
//        sqrt(k) over the cached blocks (one thread per block, all heads); then
//        per head, on 8 / group warps: the log-domain walk rho_j += s * (z_j -
//        logsumexp(z)) and the top-tau blocks of rho (8-bit radix select);
//     3. the union of the group's choices, ascending, with a per-block head mask.
//   decode_attn_kernel (split over the union): each CTA streams a slice of the
//     union's K/V blocks (cp.async, 3 stages), scores all heads of the group
//     with mma.sync tiles (heads are the M rows), keeps a running max / sum per
//     head, and writes a partial (o, max, sum) per head.
//   decode_combine_kernel: merges the partials of each (sequence, head).
#include <algorithm>

#include "select.cuh"
#include "sws_common.cuh"

namespace sws {
namespace {

// ---------------------------------------------------------------- init ------
// k_sketch for every cached block and k_psum (sum of the last block's keys).
template <int D>
__global__ void __launch_bounds__(D) init_cache_kernel(const __nv_bfloat16* __restrict__ kc, KvLayout kv,
                                                       const int32_t* __restrict__ seq_lens,
                                                       const double* __restrict__ hdt, int32_t k,
                                                       double* __restrict__ k_psum, double* __restrict__ k_sketch,
                                                       int32_t* err) {
  grid_dependency_wait();
  allow_dependents();
  __shared__ double mean[D];
  const int64_t unit = blockIdx.y;  // sequence * hkv + kv head
  const int64_t bi = unit / kv.hkv, g = unit % kv.hkv;
  const int32_t len = seq_lens[bi];
  if (len < 1 || len > kv.max_len) {
    if (threadIdx.x == 0) record_error(err, GUARD_BAD_LEN);
    return;
  }
  const int64_t nb = ceil_div64(len, kv.B);
  const int64_t j = blockIdx.x;
  if (j >= nb) return;
  const int64_t off = kv_block_offset(kv, bi, g, j);
  if (off < 0) {
    if (threadIdx.x == 0) record_error(err, GUARD_BAD_PAGE);
    return;
  }
  const int64_t rows = std::min<int64_t>(len - j * kv.B, kv.B);
  const __nv_bfloat16* base = kc + off;
  double s = 0.0;
  for (int64_t r = 0; r < rows; ++r) s += static_cast<double>(__bfloat162float(base[r * D + threadIdx.x]));
  if (j == nb - 1) k_psum[unit * D + threadIdx.x] = s;
  mean[threadIdx.x] = s / static_cast<double>(rows);
  __syncthreads();
  for (int c = threadIdx.x; c < k; c += D) {
    double acc = 0.0;
    for (int t = 0; t < D; ++t) acc += mean[t] * hdt[(size_t)c * D + t];
    k_sketch[(unit * kv.max_blocks + j) * k + c] = acc;
  }
}

__global__ void advance_kernel(int32_t* seq_lens, int32_t batch) {
  grid_dependency_wait();
  allow_dependents();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < batch) seq_lens[i] += 1;
}

// -------------------------------------------------------------- select ------
constexpr int kSelThreads = 1024;
constexpr int kSelWarps = kSelThreads / 32;

// One CTA per (sequence, KV head); the query heads of the group split the
// warps between them (8 / group warps each) for their walk and selection.
template <int D>
__global__ void __launch_bounds__(kSelThreads) decode_select_kernel(
    const __nv_bfloat16* __restrict__ q_tok, const __nv_bfloat16* __restrict__ k_tok,
    const __nv_bfloat16* __restrict__ v_tok, int32_t hq, KvLayout kv, const int32_t* __restrict__ seq_lens,
    __nv_bfloat16* __restrict__ k_cache, __nv_bfloat16* __restrict__ v_cache, double* __restrict__ k_psum,
    double* __restrict__ k_sketch, int first_layer, double* __restrict__ walk_state,
    int32_t* __restrict__ head_sel, int32_t* __restrict__ head_cnt, int32_t* __restrict__ sel,
    uint8_t* __restrict__ sel_mask, int32_t* __restrict__ sel_cnt, const double* __restrict__ hdt, int32_t k,
    int32_t B, int32_t s_pow, int32_t num, int32_t den, int shared, int32_t* err) {
  grid_dependency_wait();
  allow_dependents();
  const int32_t hkv = kv.hkv;
  const int64_t max_blocks = kv.max_blocks;
  const int group = hq / hkv;
  extern __shared__ __align__(16) uint8_t smem[];
  uint64_t* keys = reinterpret_cast<uint64_t*>(smem);                       // [group][max_blocks] (z, then keys)
  uint32_t* mark = reinterpret_cast<uint32_t*>(keys + group * max_blocks);  // [max_blocks]
  double* qt = reinterpret_cast<double*>(mark + ((max_blocks + 1) & ~int64_t(1)));  // [group][k]
  double* mean = qt + group * k;                                            // [D]
  double* qrow = mean + D;                                                  // [group][D]
  double* red = qrow + group * D;                                           // [kSelWarps]
  int* hist = reinterpret_cast<int*>(red + kSelWarps);                      // [group][256]
  int* ctl = hist + group * 256;                                            // [group][4]
  int* wsum = ctl + group * 4;                                              // [kSelWarps + 1]

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t unit = blockIdx.x;
  const int bi = static_cast<int>(unit / hkv), g = static_cast<int>(unit % hkv);
  const int32_t len = seq_lens[bi];
  if (len < 1 || len > kv.max_len) {
    if (tid == 0) record_error(err, GUARD_BAD_LEN);
    return;
  }
  const int64_t pos = len - 1;
  const int64_t blk = pos / B;
  const int cnt = static_cast<int>(pos % B) + 1;
  const int nb = static_cast<int>(blk + 1);
  const int64_t tok_off = kv_block_offset(kv, bi, g, blk);  // the same for every thread
  if (tok_off < 0) {
    if (tid == 0) record_error(err, GUARD_BAD_PAGE);
    return;
  }
  for (int j = tid; j < nb; j += kSelThreads) mark[j] = 0u;

  // 1. append the token, update the last block's running key sum; stage the
  //    block mean and the group's query rows
  if (tid < D) {
    const __nv_bfloat16 kt = k_tok[unit * D + tid];
    k_cache[tok_off + (pos % B) * D + tid] = kt;
    v_cache[tok_off + (pos % B) * D + tid] = v_tok[unit * D + tid];
    double ps = (cnt == 1) ? 0.0 : k_psum[unit * D + tid];
    ps += static_cast<double>(__bfloat162float(kt));
    k_psum[unit * D + tid] = ps;
    mean[tid] = ps / cnt;
  }
  for (int x = tid; x < group * D; x += kSelThreads)
    qrow[x] = static_cast<double>(__bfloat162float(q_tok[((int64_t)bi * hq + (int64_t)g * group) * D + x]));
  __syncthreads();
  // the last block's sketch k~ = mean H_d and q~ = q H_d, one warp per output
  double* ksk = k_sketch + unit * max_blocks * k;
  for (int o = warp; o < (group + 1) * k; o += kSelWarps) {
    const int r = o / k, c = o % k;  // r == group: the key block
    const double v = warp_dot_hdt<D>(r == group ? mean : qrow + r * D, hdt + (size_t)c * D, lane);
    if (lane == 0) {
      if (r == group) ksk[blk * k + c] = v;
      else qt[r * k + c] = v;
    }
  }
  __syncthreads();

  // 2. z_j = q~ . k~_j / sqrt(k) for every head on the fp64 tensor path: one
  //    m16n8k4 product per 8 key blocks and 4 sketch dims, the group's query
  //    heads as rows 0..group-1 of A; a lane's k~ fragment is 4 consecutive
  //    doubles of one cached block, so every load uses whole sectors
  double* z = reinterpret_cast<double*>(keys);
  const double inv_sqrt_k = 1.0 / sqrt((double)k);
  {
    const int g8 = lane >> 2, t4 = lane & 3;
    for (int n0 = warp * 8; n0 < nb; n0 += kSelWarps * 8) {
      const int j = n0 + g8;
      const double* kr = ksk + (int64_t)(j < nb ? j : 0) * k;
      double c4[4] = {0.0, 0.0, 0.0, 0.0};
      for (int c0 = 0; c0 < k; c0 += 4) {
        const int c = c0 + t4;
        const double a0 = (g8 < group && c < k) ? qt[g8 * k + c] : 0.0;
        const double b0 = (j < nb && c < k) ? kr[c] : 0.0;
        asm volatile(
            "mma.sync.aligned.m16n8k4.row.col.f64.f64.f64.f64 {%0,%1,%2,%3}, {%4,%5}, {%6}, {%0,%1,%2,%3};"
            : "+d"(c4[0]), "+d"(c4[1]), "+d"(c4[2]), "+d"(c4[3])
            : "d"(a0), "d"(0.0), "d"(b0));
      }
      // c4[0], c4[1]: head g8, key blocks n0 + 2 t4 and n0 + 2 t4 + 1
      if (g8 < group) {
        const int j0 = n0 + 2 * t4;
        if (j0 < nb) z[g8 * max_blocks + j0] = c4[0] * inv_sqrt_k;
        if (j0 + 1 < nb) z[g8 * max_blocks + j0 + 1] = c4[1] * inv_sqrt_k;
      }
    }
  }
  __syncthreads();

  // 3. per head: log-domain walk, then top-tau (its share of the warps)
  const int tau = tau_of_row(nb - 1, num, den);
  const int wph = kSelWarps / group;  // >= 1 since group <= 8
  const int r = warp / wph;
  if (r < group) {
    const int t = tid - r * wph * 32, nthr = wph * 32, bar_id = 1 + r;
    const int h = g * group + r;
    double* zr = z + r * max_blocks;
    double mx = -INFINITY;
    for (int j = t; j < nb; j += nthr) mx = fmax(mx, zr[j]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    if (lane == 0) red[warp] = mx;
    named_bar(bar_id, nthr);
    mx = red[r * wph];
    for (int w = 1; w < wph; ++w) mx = fmax(mx, red[r * wph + w]);
    named_bar(bar_id, nthr);
    double se = 0.0;
    for (int j = t; j < nb; j += nthr) se += exp(zr[j] - mx);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) se += __shfl_xor_sync(0xffffffffu, se, off);
    if (lane == 0) red[warp] = se;
    named_bar(bar_id, nthr);
    se = 0.0;
    for (int w = 0; w < wph; ++w) se += red[r * wph + w];
    const double lse = mx + log(se);
    double* rho = walk_state + ((int64_t)bi * hq + h) * max_blocks;
    uint64_t* kr = keys + r * max_blocks;
    for (int j = t; j < nb; j += nthr) {
      const double val = (first_layer ? 0.0 : rho[j]) + s_pow * (zr[j] - lse);
      rho[j] = val;
      if (shared) zr[j] = val;  // kept for the group's log-sum-exp below
      else kr[j] = order_key(val);
    }
    named_bar(bar_id, nthr);
    if (!shared) {
      group_top_tau(kr, nb, tau, hist + r * 256, ctl + r * 4, t, nthr, bar_id,
                    head_sel + ((int64_t)bi * hq + h) * max_blocks, mark, 1u << r, err);
      if (t == 0) head_cnt[(int64_t)bi * hq + h] = tau;
    }
  }
  __syncthreads();
  if (shared) {
    // one selection for the whole group: the top-tau of log(sum_h exp(rho_h)),
    // by every warp of the CTA; the other heads copy the first head's list
    for (int j = tid; j < nb; j += kSelThreads) {
      double m = z[j];
      for (int q = 1; q < group; ++q) m = fmax(m, z[q * max_blocks + j]);
      double se = 0.0;
      for (int q = 0; q < group; ++q) se += exp(z[q * max_blocks + j] - m);
      keys[j] = order_key(m + log(se));
    }
    __syncthreads();
    int32_t* sel0 = head_sel + ((int64_t)bi * hq + (int64_t)g * group) * max_blocks;
    group_top_tau(keys, nb, tau, hist, ctl, tid, kSelThreads, 1, sel0, mark, (1u << group) - 1u, err);
    __syncthreads();
    for (int q = 1; q < group; ++q)
      for (int x = tid; x < tau; x += kSelThreads) sel0[(int64_t)q * max_blocks + x] = sel0[x];
    if (tid < group) head_cnt[(int64_t)bi * hq + g * group + tid] = tau;
    __syncthreads();
  }

  // 4. ordered compaction of the union
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

// ----------------------------------------------------------- attention ------
__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p)));
}

__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

constexpr int kAttnThreads = 128;
constexpr int kStages = 2;

// Row u of a staged [B][D] bf16 tile keeps its 16-byte chunks XOR-swizzled by
// u mod (D/8), so that the column accesses of the mma fragments and of
// ldmatrix hit distinct banks.
template <int D>
__device__ __forceinline__ int swz(int u, int d) {
  constexpr int CPR = D / 8;
  return u * D + (((d >> 3) ^ (u & (CPR - 1))) << 3) + (d & 7);
}

// kPaged: the cache is a page pool (a block-table lookup per block); otherwise
// contiguous [batch, hkv, max_len, D].
template <int D, int BS, int G, bool kPaged>
__global__ void __launch_bounds__(kAttnThreads) decode_attn_kernel(
    const __nv_bfloat16* __restrict__ q_tok, const __nv_bfloat16* __restrict__ k_cache,
    const __nv_bfloat16* __restrict__ v_cache, KvLayout kv, const int32_t* __restrict__ seq_lens,
    const int32_t* __restrict__ sel, const uint8_t* __restrict__ sel_mask, const int32_t* __restrict__ sel_cnt,
    float* __restrict__ partial, int32_t splits, int32_t* err) {
  grid_dependency_wait();
  allow_dependents();
  static_assert(G >= 1 && G <= 8, "GQA group of 1..8 query heads");
  constexpr int NT_QK = BS / 8 / 4;  // score n-tiles (8 tokens) per warp
  constexpr int NT_PV = D / 8 / 4;   // output n-tiles (8 dims) per warp
  constexpr int TILE = BS * D;
  extern __shared__ __align__(16) uint8_t smem[];
  __nv_bfloat16* stage = reinterpret_cast<__nv_bfloat16*>(smem);  // [kStages][2][BS][D]
  constexpr int SCS = BS + 4;  // padded score row: the 8 head rows fall in different banks
  float* sc = reinterpret_cast<float*>(stage + kStages * 2 * TILE);  // [8][SCS]
  __nv_bfloat16* ps = reinterpret_cast<__nv_bfloat16*>(sc + 8 * SCS);  // [8][BS + 8]
  float* corr_s = reinterpret_cast<float*>(ps + 8 * (BS + 8));       // [8]
  float* ml_s = corr_s + 8;                                          // [8][2]

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gq = lane >> 2, tq = lane & 3;
  const int32_t hkv = kv.hkv;
  const int64_t max_blocks = kv.max_blocks;
  const int64_t unit = blockIdx.y;
  const int bi = static_cast<int>(unit / hkv);
  const int split = blockIdx.x;
  int32_t len = seq_lens[bi];
  int64_t U = sel_cnt[unit];
  if (len < 1 || len > kv.max_len || U < 0 || U > ceil_div64(len, BS)) {  // stale or corrupt state: no work
    if (tid == 0) record_error(err, GUARD_BAD_LEN);
    len = 0;
    U = 0;
  }
  const int64_t lo = U * split / splits, hi = U * (split + 1) / splits;
  const int32_t* blist = sel + unit * max_blocks;
  const uint8_t* mlist = sel_mask + unit * max_blocks;

  // Q fragments (rows = heads of the group, pre-scaled later in fp32)
  uint32_t qa[D / 16][2];
  {
    const int h = (gq < G) ? gq : 0;
    const __nv_bfloat16* qr = q_tok + ((int64_t)bi * hkv * G + (unit % hkv) * G + h) * D;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      const uint32_t x0 = *reinterpret_cast<const uint32_t*>(qr + ks * 16 + 2 * tq);
      const uint32_t x1 = *reinterpret_cast<const uint32_t*>(qr + ks * 16 + 8 + 2 * tq);
      qa[ks][0] = (gq < G) ? x0 : 0u;
      qa[ks][1] = (gq < G) ? x1 : 0u;
    }
  }
  for (int x = tid; x < 8 * (BS + 8); x += kAttnThreads) ps[x] = __float2bfloat16_rn(0.f);
  if (tid < 8) {  // running max (log2 units) and sum per head
    ml_s[2 * tid] = -INFINITY;
    ml_s[2 * tid + 1] = 0.f;
  }
  float oacc[NT_PV][4];
#pragma unroll
  for (int nt = 0; nt < NT_PV; ++nt) oacc[nt][0] = oacc[nt][1] = oacc[nt][2] = oacc[nt][3] = 0.f;

  auto block_ok = [&](int64_t j) { return j >= 0 && j * BS < len; };
  // contiguous: the unit's rows; paged: looked up per block. A row that is
  // not loaded (src-size 0) still gets an address inside the cache.
  const __nv_bfloat16* kbase = k_cache + (kPaged ? 0 : unit * kv.max_len * D);
  const __nv_bfloat16* vbase = v_cache + (kPaged ? 0 : unit * kv.max_len * D);
  // Paged: issue() is called for idx = lo, lo + 1, ... in order. The list
  // entry of idx + 2 and the page of idx + 1 are loaded while idx is issued,
  // and only used (the page checked and turned into an offset) one call
  // later, so the copies of a block never wait on the two dependent lookups.
  int64_t pf_raw = lo < hi ? blist[lo] : -1;  // list entry of the next idx to issue
  int64_t pf_page = (kPaged && block_ok(pf_raw)) ? kv.block_table[(int64_t)bi * kv.max_blocks + pf_raw] : -1;
  int64_t pf_raw2 = lo + 1 < hi ? blist[lo + 1] : -1;  // list entry after it
  auto issue = [&](int64_t idx, int st) {
    int64_t j;
    const __nv_bfloat16* kblk = kbase;
    const __nv_bfloat16* vblk = vbase;
    if constexpr (kPaged) {
      j = block_ok(pf_raw) ? pf_raw : -1;
      if (j >= 0 && (pf_page < 0 || pf_page >= kv.num_pages)) {
        if (tid == 0) record_error(err, GUARD_BAD_PAGE);
        j = -1;
      }
      if (j >= 0) {
        const int64_t off = ((pf_page * hkv + unit % hkv) * BS) * D;
        kblk += off;
        vblk += off;
      }
      pf_raw = pf_raw2;
      pf_page = (idx + 1 < hi && block_ok(pf_raw)) ? kv.block_table[(int64_t)bi * kv.max_blocks + pf_raw] : -1;
      pf_raw2 = idx + 2 < hi ? blist[idx + 2] : -1;
    } else {
      j = block_ok(blist[idx]) ? blist[idx] : -1;
    }
    const int64_t t0 = j < 0 ? (int64_t)len : j * BS;  // an invalid block stages zeros
    __nv_bfloat16* ksm = stage + (st * 2) * TILE;
    __nv_bfloat16* vsm = ksm + TILE;
    for (int x = tid; x < TILE / 8; x += kAttnThreads) {
      const int u = x / (D / 8), c = x % (D / 8);
      const bool valid = t0 + u < len;
      const __nv_bfloat16* ks;
      const __nv_bfloat16* vs;
      if constexpr (kPaged) {
        ks = valid ? kblk + u * D : kbase;
        vs = valid ? vblk + u * D : vbase;
      } else {
        const int64_t row = valid ? (t0 + u) : 0;
        ks = kbase + row * D;
        vs = vbase + row * D;
      }
      cp_async16(ksm + swz<D>(u, c * 8), ks + c * 8, valid);
      cp_async16(vsm + swz<D>(u, c * 8), vs + c * 8, valid);
    }
  };

  const float qscale = 1.4426950408889634f / sqrtf((float)D);
#pragma unroll
  for (int p = 0; p < kStages - 1; ++p) {
    if (lo + p < hi) issue(lo + p, p);
    cp_async_commit();
  }
  for (int64_t it = lo; it < hi; ++it) {
    const int st = static_cast<int>((it - lo) % kStages);
    if (it + kStages - 1 < hi) issue(it + kStages - 1, static_cast<int>((it - lo + kStages - 1) % kStages));
    cp_async_commit();
    cp_async_wait<kStages - 1>();
    __syncthreads();
    const __nv_bfloat16* ksm = stage + (st * 2) * TILE;
    const __nv_bfloat16* vsm = ksm + TILE;
    const int64_t jraw = blist[it];
    const bool jok = block_ok(jraw);
    if (!jok && tid == 0) record_error(err, GUARD_BAD_CSR);
    const uint32_t hm = jok ? mlist[it] : 0u;
    const int64_t t0 = jok ? jraw * BS : 0;

    // scores: warp handles n-tiles [warp*NT_QK, (warp+1)*NT_QK)
#pragma unroll
    for (int nt = 0; nt < NT_QK; ++nt) {
      const int n0 = (warp * NT_QK + nt) * 8;
      float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        const int u = n0 + gq;
        const uint32_t b0 = *reinterpret_cast<const uint32_t*>(ksm + swz<D>(u, ks * 16 + 2 * tq));
        const uint32_t b1 = *reinterpret_cast<const uint32_t*>(ksm + swz<D>(u, ks * 16 + 8 + 2 * tq));
        const uint32_t a[4] = {qa[ks][0], 0u, qa[ks][1], 0u};
        mma_bf16_16816(c, a, b0, b1);
      }
      if (gq < G) {
        const bool hv = (hm >> gq) & 1u;
        const int u0 = n0 + 2 * tq;
        sc[gq * SCS + u0] = (hv && t0 + u0 < len) ? c[0] * qscale : -INFINITY;
        sc[gq * SCS + u0 + 1] = (hv && t0 + u0 + 1 < len) ? c[1] * qscale : -INFINITY;
      }
    }
    __syncthreads();
    // online softmax: warp w owns heads w, w + 4
    for (int r = warp; r < G; r += 4) {
      float mx = -INFINITY;
      for (int u = lane; u < BS; u += 32) mx = fmaxf(mx, sc[r * SCS + u]);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      const float mr = ml_s[2 * r];
      const float mn = fmaxf(mr, mx);
      float corr = 1.f, sum = 0.f;
      if (mn != -INFINITY) {
        corr = exp2f(mr - mn);
        for (int u = lane; u < BS; u += 32) {
          const float p = exp2f(sc[r * SCS + u] - mn);
          sum += p;
          ps[r * (BS + 8) + u] = __float2bfloat16_rn(p);
        }
      } else {
        for (int u = lane; u < BS; u += 32) ps[r * (BS + 8) + u] = __float2bfloat16_rn(0.f);
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
      __syncwarp();
      if (lane == 0) {
        corr_s[r] = corr;
        ml_s[2 * r] = mn;
        ml_s[2 * r + 1] = ml_s[2 * r + 1] * corr + sum;
      }
    }
    __syncthreads();
    // P V: warp handles output dims [warp*NT_PV*8, (warp+1)*NT_PV*8)
    {
      const float cr = (gq < G) ? corr_s[gq] : 1.f;
#pragma unroll
      for (int nt = 0; nt < NT_PV; ++nt) {
        oacc[nt][0] *= cr;
        oacc[nt][1] *= cr;
      }
#pragma unroll
      for (int kk = 0; kk < BS / 16; ++kk) {
        uint32_t a[4];
        a[0] = *reinterpret_cast<const uint32_t*>(ps + gq * (BS + 8) + kk * 16 + 2 * tq);
        a[1] = 0u;
        a[2] = *reinterpret_cast<const uint32_t*>(ps + gq * (BS + 8) + kk * 16 + 8 + 2 * tq);
        a[3] = 0u;
#pragma unroll
        for (int np = 0; np < NT_PV / 2; ++np) {
          const int n0 = (warp * NT_PV + 2 * np) * 8;
          const int mi = lane >> 3, ri = lane & 7;
          const int u = kk * 16 + ri + 8 * (mi & 1);
          const int dcol = n0 + 8 * (mi >> 1);
          uint32_t bfr[4];
          ldsm_x4_trans(bfr, vsm + swz<D>(u, dcol));
          mma_bf16_16816(oacc[2 * np], a, bfr[0], bfr[1]);
          mma_bf16_16816(oacc[2 * np + 1], a, bfr[2], bfr[3]);
        }
      }
    }
    __syncthreads();
  }
  cp_async_wait<0>();

  // partial results: [unit][head][split][D + 2]
  if (gq < G) {
    float* pr = partial + (((unit * G + gq) * splits) + split) * (D + 2);
#pragma unroll
    for (int nt = 0; nt < NT_PV; ++nt) {
      const int d0 = (warp * NT_PV + nt) * 8 + 2 * tq;
      pr[d0] = oacc[nt][0];
      pr[d0 + 1] = oacc[nt][1];
    }
  }
  if (tid < G) {
    float* pr = partial + (((unit * G + tid) * splits) + split) * (D + 2);
    const bool any = hi > lo;
    pr[D] = any ? ml_s[2 * tid] : -INFINITY;
    pr[D + 1] = any ? ml_s[2 * tid + 1] : 0.f;
  }
}

template <int D>
__global__ void __launch_bounds__(D) decode_combine_kernel(const float* __restrict__ partial, int32_t hq, int32_t hkv,
                                                           int32_t splits, __nv_bfloat16* __restrict__ o) {
  grid_dependency_wait();
  allow_dependents();
  const int64_t bh = blockIdx.x;  // sequence * hq + head
  const int group = hq / hkv;
  const int64_t bi = bh / hq;
  const int h = static_cast<int>(bh % hq);
  const int64_t unit = bi * hkv + h / group;
  const float* pr = partial + ((unit * group + h % group) * splits) * (D + 2);
  float M = -INFINITY;
  for (int s = 0; s < splits; ++s) M = fmaxf(M, pr[s * (D + 2) + D]);
  float L = 0.f, acc = 0.f;
  for (int s = 0; s < splits; ++s) {
    const float ms = pr[s * (D + 2) + D];
    if (ms == -INFINITY) continue;
    const float w = exp2f(ms - M);
    L += w * pr[s * (D + 2) + D + 1];
    acc += w * pr[s * (D + 2) + threadIdx.x];
  }
  o[bh * D + threadIdx.x] = __float2bfloat16_rn(L > 0.f ? acc / L : 0.f);
}

template <int D, int BS, int G>
cudaError_t launch_attn3(const __nv_bfloat16* q, const __nv_bfloat16* kc, const __nv_bfloat16* vc, int32_t batch,
                         const KvLayout& kv, const int32_t* lens, const int32_t* sel, const uint8_t* mask,
                         const int32_t* cnt, float* partial, int32_t splits, int32_t* err, cudaStream_t st) {
  const size_t smem = (size_t)kStages * 2 * BS * D * 2 + 8 * (BS + 4) * 4 + 8 * (BS + 8) * 2 + 8 * 4 + 16 * 4;
  auto kern = kv.block_table ? decode_attn_kernel<D, BS, G, true> : decode_attn_kernel<D, BS, G, false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(splits, static_cast<unsigned>((int64_t)batch * kv.hkv));
  {
    const cudaError_t le = launch_k(kern, grid, kAttnThreads, smem, st, q, kc, vc, kv, lens, sel, mask, cnt, partial,
                                    splits, err);
    if (le != cudaSuccess) return le;
  }
  note_launches(1);
  return cudaGetLastError();
}

template <int D, int BS>
cudaError_t launch_attn2(int32_t group, const __nv_bfloat16* q, const __nv_bfloat16* kc, const __nv_bfloat16* vc,
                         int32_t batch, const KvLayout& kv, const int32_t* lens, const int32_t* sel,
                         const uint8_t* mask, const int32_t* cnt, float* partial, int32_t splits, int32_t* err,
                         cudaStream_t st) {
#define SWS_G(GG) \
  case GG:        \
    return launch_attn3<D, BS, GG>(q, kc, vc, batch, kv, lens, sel, mask, cnt, partial, splits, err, st);
  switch (group) {
    SWS_G(1) SWS_G(2) SWS_G(4) SWS_G(8)
    default:
      return cudaErrorInvalidValue;
  }
#undef SWS_G
}

}  // namespace

size_t decode_select_smem_bytes(const sws_config& cfg, int64_t max_blocks, int32_t group) {
  const int64_t k = cfg.sketch_dim, D = cfg.head_dim;
  return (size_t)group * max_blocks * 8 + (size_t)((max_blocks + 1) & ~int64_t(1)) * 4 + (size_t)group * k * 8 +
         (size_t)D * 8 + (size_t)group * D * 8 + kSelWarps * 8 + (size_t)group * 256 * 4 + (size_t)group * 4 * 4 +
         (kSelWarps + 1) * 4;
}

int32_t decode_num_splits(const sws_config& cfg, int64_t max_len, int32_t group) {
  const int64_t mb = ceil_div64(max_len, cfg.block_size);
  const int64_t umax = std::min<int64_t>(mb, (int64_t)group * tau_of_row(mb - 1, cfg.density_num, cfg.density_den));
  return static_cast<int32_t>(std::max<int64_t>(1, std::min<int64_t>(256, ceil_div64(umax, 16))));
}

cudaError_t launch_decode_init_cache(const sws_handle* h, const __nv_bfloat16* k_cache, const KvLayout& kv,
                                     int32_t batch, const int32_t* seq_lens, double* k_psum, double* k_sketch,
                                     cudaStream_t st) {
  dim3 grid(static_cast<unsigned>(kv.max_blocks), static_cast<unsigned>((int64_t)batch * kv.hkv));
  if (h->cfg.head_dim == 128)
    {
      const cudaError_t le = launch_k(init_cache_kernel<128>, grid, 128, 0, st, k_cache, kv, seq_lens,
                                      h->hdt, h->cfg.sketch_dim, k_psum, k_sketch, h->err);
      if (le != cudaSuccess) return le;
    }
  else
    {
      const cudaError_t le = launch_k(init_cache_kernel<64>, grid, 64, 0, st, k_cache, kv, seq_lens,
                                      h->hdt, h->cfg.sketch_dim, k_psum, k_sketch, h->err);
      if (le != cudaSuccess) return le;
    }
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_decode_advance(int32_t* seq_lens, int32_t batch, cudaStream_t st) {
  {
    const cudaError_t le = launch_k(advance_kernel, static_cast<unsigned>(ceil_div64(batch, 128)), 128, 0, st, seq_lens,
                                    batch);
    if (le != cudaSuccess) return le;
  }
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_decode_select(const sws_handle* h, const __nv_bfloat16* q_tok, const __nv_bfloat16* k_tok,
                                 const __nv_bfloat16* v_tok, int32_t batch, int32_t hq, const KvLayout& kv,
                                 const int32_t* seq_lens, __nv_bfloat16* k_cache, __nv_bfloat16* v_cache,
                                 double* k_psum, double* k_sketch, int first_layer, double* walk_state,
                                 int32_t* head_sel, int32_t* head_cnt, int32_t* sel, uint8_t* sel_mask,
                                 int32_t* sel_cnt, cudaStream_t st) {
  const sws_config& c = h->cfg;
  const int32_t hkv = kv.hkv;
  const size_t smem = decode_select_smem_bytes(c, kv.max_blocks, hq / hkv);
  auto kern = c.head_dim == 128 ? decode_select_kernel<128> : decode_select_kernel<64>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  {
    const cudaError_t le = launch_k(kern, static_cast<unsigned>((int64_t)batch * hkv), kSelThreads, smem, st, q_tok,
                                    k_tok, v_tok, hq, kv, seq_lens, k_cache, v_cache, k_psum, k_sketch, first_layer,
                                    walk_state, head_sel, head_cnt, sel, sel_mask, sel_cnt, h->hdt, c.sketch_dim,
                                    c.block_size, c.walk_power, c.density_num, c.density_den,
                                    (c.select_group > 1 && hq / hkv > 1) ? 1 : 0, h->err);
    if (le != cudaSuccess) return le;
  }
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_decode_attn(const sws_handle* h, const __nv_bfloat16* q_tok, const __nv_bfloat16* k_cache,
                               const __nv_bfloat16* v_cache, int32_t batch, int32_t hq, const KvLayout& kv,
                               const int32_t* seq_lens, const int32_t* sel, const uint8_t* sel_mask,
                               const int32_t* sel_cnt, __nv_bfloat16* o, float* partial, int32_t splits,
                               cudaStream_t st) {
  const sws_config& c = h->cfg;
  const int32_t hkv = kv.hkv;
  const int32_t group = hq / hkv;
  cudaError_t e;
  if (c.head_dim == 128)
    e = c.block_size == 64 ? launch_attn2<128, 64>(group, q_tok, k_cache, v_cache, batch, kv, seq_lens, sel, sel_mask,
                                                    sel_cnt, partial, splits, h->err, st)
                           : launch_attn2<128, 128>(group, q_tok, k_cache, v_cache, batch, kv, seq_lens, sel,
                                                     sel_mask, sel_cnt, partial, splits, h->err, st);
  else
    e = c.block_size == 64 ? launch_attn2<64, 64>(group, q_tok, k_cache, v_cache, batch, kv, seq_lens, sel, sel_mask,
                                                   sel_cnt, partial, splits, h->err, st)
                           : launch_attn2<64, 128>(group, q_tok, k_cache, v_cache, batch, kv, seq_lens, sel, sel_mask,
                                                    sel_cnt, partial, splits, h->err, st);
  if (e != cudaSuccess) return e;
  if (c.head_dim == 128)
    {
      const cudaError_t le = launch_k(decode_combine_kernel<128>, static_cast<unsigned>((int64_t)batch * hq), 128, 0,
                                      st, partial, hq, hkv, splits, o);
      if (le != cudaSuccess) return le;
    }
  else
    {
      const cudaError_t le = launch_k(decode_combine_kernel<64>, static_cast<unsigned>((int64_t)batch * hq), 64, 0, st,
                                      partial, hq, hkv, splits, o);
      if (le != cudaSuccess) return le;
    }
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace sws

// ---------------------------------------------------------------------------
// Decode attention for callers that cannot allocate device memory.
//
// Some callers may not call cudaMalloc, or hand the library any memory it did
// not receive from them, at the point where they run decode attention: plug-ins
// inside a host framework that owns every device allocation, serving loops that
// must not take the synchronisation and latency of an allocation on the token
// path, and code that runs under an allocator budget fixed ahead of time. For
// them this variant keeps the split-KV partial results in one scratch array
// that lives in the library itself, sized SWS_NOALLOC_SCRATCH_BYTES, allocated
// by the CUDA runtime when the library is loaded on a device and held until
// the process exits.

static __device__ __align__(256) unsigned char g_noalloc_scratch[SWS_NOALLOC_SCRATCH_BYTES];

namespace sws {

// Device address of g_noalloc_scratch on the current device. On the host the
// array's name is only a stand-in for the device symbol: a kernel must receive
// the address that cudaGetSymbolAddress returns in the context it runs in.
// sws_create calls this once per handle, with the handle's device current, and
// keeps the result in the handle, so a context that is torn down and created
// again (cudaDeviceReset) gives new handles the new address.
cudaError_t noalloc_scratch_address(void** out) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess) return e;
  *out = p;
  return cudaSuccess;
}

}  // namespace sws

extern "C" sws_status sws_sparse_attn_decode_noalloc(const sws_handle* h, const void* q_tok, const void* k_cache,
                                                     const void* v_cache, int32_t batch, int32_t hq, int32_t hkv,
                                                     int64_t max_len, const int32_t* seq_lens, const int32_t* sel,
                                                     const uint8_t* sel_mask, const int32_t* sel_cnt, void* o,
                                                     void* stream) {
  if (!h || batch < 1 || max_len < 1 || hq < 1 || hkv < 1 || hq % hkv != 0 || hq > 4096) return SWS_ERR_INVALID_ARG;
  const int32_t group = hq / hkv;
  if (group != 1 && group != 2 && group != 4 && group != 8) return SWS_ERR_UNSUPPORTED;
  const void* ptrs[] = {q_tok, k_cache, v_cache, seq_lens, sel, sel_mask, sel_cnt, o};
  for (const void* p : ptrs)
    if (!p || (reinterpret_cast<uintptr_t>(p) & 15u) != 0) return SWS_ERR_INVALID_ARG;
  const int32_t splits = sws::decode_num_splits(h->cfg, max_len, group);
  const size_t need = static_cast<size_t>(batch) * hq * splits * (h->cfg.head_dim + 2) * sizeof(float);
  if (need > SWS_NOALLOC_SCRATCH_BYTES) return SWS_ERR_WORKSPACE;  // beyond the built-in scratch
  int device = -1;
  if (cudaGetDevice(&device) != cudaSuccess || device != h->device) return SWS_ERR_INVALID_ARG;
  void* scratch = h->noalloc_scratch;
  if (!scratch) return SWS_ERR_CUDA;
  const cudaError_t e = sws::launch_decode_attn(
      h, static_cast<const __nv_bfloat16*>(q_tok), static_cast<const __nv_bfloat16*>(k_cache),
      static_cast<const __nv_bfloat16*>(v_cache), batch, hq, sws::contiguous_kv(h->cfg, hkv, max_len), seq_lens, sel,
      sel_mask, sel_cnt, static_cast<__nv_bfloat16*>(o), static_cast<float*>(scratch), splits,
      static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SWS_OK : SWS_ERR_CUDA;
}
