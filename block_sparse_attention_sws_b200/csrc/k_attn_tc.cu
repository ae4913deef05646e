// sw_sparse_attn_prefill on the 5th-generation tensor cores (bf16 in, fp32 accumulate).
//
// "Scout Before You Attend" §4/§5: exact softmax attention on the original
// Q, K, V restricted to the key blocks selected for each query block (query
// token t sees key token u of a selected block iff u <= t).
//
// One persistent CTA per SM walks (head, 128-row query tile) work items, longest
// first. A tile is one query block (B = 128) or two adjacent query blocks
// (B = 64, whose selections overlap almost entirely): their CSR rows are merged
// and consecutive key blocks of the union are paired into 128-key tiles with a
// per-(query half, key half) selection mask.
//
// Warp roles (192 threads):
//   warp 0    TMA producer: Q tile once per item, K and V tiles into a 2-stage
//             ring (3-D tensor maps, 128-byte swizzle, zero fill past n);
//   warp 1    owns 512 TMEM columns and issues tcgen05.mma from one thread:
//             S = Q K^T into one of two TMEM S buffers, then O += P V;
//   warps 2-5 softmax, one query row per thread (TMEM lane = row): reads S,
//             masks, keeps a running max that is only moved when it grows by
//             more than 2^8 (then the row of O in TMEM is rescaled), writes
//             P = 2^(s - m) as bf16 into one of two swizzled shared buffers,
//             and finally writes O / l.
// Every wait is bounded; a timeout records a guard code and all roles leave.
#include <cuda.h>

#include <algorithm>

#include "sws_common.cuh"

namespace sws {
namespace {

constexpr int kTcThreads = 192;
constexpr int kTileM = 128;  // query rows per item
constexpr int kTileN = 128;  // keys per S tile
constexpr float kRescaleLog2 = 8.0f;

// ---- PTX wrappers --------------------------------------------------------------

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int x, int y, int z, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
      "[%5];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tc_mma(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Loads 32 consecutive columns of this thread's TMEM lane; the wait for the
// load sits in the same statement, so the registers are valid on return.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%"
      "19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%"
      "18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])),
      "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])),
      "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])),
      "r"(__float_as_uint(v[11])), "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])),
      "r"(__float_as_uint(v[14])), "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])),
      "r"(__float_as_uint(v[17])), "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])),
      "r"(__float_as_uint(v[20])), "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])),
      "r"(__float_as_uint(v[23])), "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])),
      "r"(__float_as_uint(v[26])), "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])),
      "r"(__float_as_uint(v[29])), "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Shared-memory matrix descriptor, 128-byte swizzle (sm_100 "version 1").
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= 1ull << 46;
  d |= 2ull << 61;
  return d;
}

// Instruction descriptor, kind::f16: bf16 A and B, fp32 D, M = 128.
__host__ __device__ constexpr uint32_t idesc_bf16(int n, bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn_major ? 1u : 0u) << 16) | (static_cast<uint32_t>(n >> 3) << 17) |
         (static_cast<uint32_t>(kTileM >> 4) << 24);
}

// ---- shared state ----------------------------------------------------------------

struct TileMeta {
  int32_t u0, u1;  // key blocks of the two key halves (B = 64) or the key block (B = 128)
  int32_t mask;    // bit (2 * key_half + query_half): that query block selected that key block
  int32_t last;    // last key tile of the item
};

struct Bars {
  uint64_t q_full, q_empty, o_empty;
  uint64_t kv_full[2], kv_empty[2];
  uint64_t s_full[2], s_empty[2];
  uint64_t p_full[2], pv_done[2];
  TileMeta meta[2];
  uint32_t tmem_base;
  volatile int32_t abort;
};

template <int D>
struct Smem {
  static constexpr uint32_t kQ = kTileM * D * 2;
  static constexpr uint32_t kK = kTileN * D * 2;
  static constexpr uint32_t kP = kTileM * kTileN * 2;
  static constexpr uint32_t q = 0;
  static constexpr uint32_t k0 = q + kQ;
  static constexpr uint32_t v0 = k0 + 2 * kK;
  static constexpr uint32_t p0 = v0 + 2 * kK;
  static constexpr uint32_t bars = p0 + 2 * kP;
  static constexpr uint32_t total = bars + sizeof(Bars);
};

// Bounded wait (wall time) that also gives up as soon as another role has aborted.
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, Bars* bs, int32_t* err) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  while (true) {
    if (mbar_try_wait_hint(bar, parity, kSuspendNs)) return true;
    if (bs->abort) return false;
    if (global_ns() - t0 > kWaitNs) break;
  }
  record_error(err, GUARD_MBAR_TIMEOUT);
  bs->abort = 1;
  return false;
}

// The softmax warps run warp-collective tcgen05.ld/st: a wait's outcome is
// made uniform across the warp before any of them.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, Bars* bs, int32_t* err) {
  return __all_sync(0xffffffffu, wait_bar(bar, parity, bs, err));
}

// Walks the key tiles of one item: for B = 128 the CSR row of query block m;
// for B = 64 the merge of rows 2m and 2m+1, two union blocks per tile.
template <int BLK>
struct TileWalker {
  const int32_t* c0;
  const int32_t* c1;
  int32_t n0, n1, p0, p1, last0, last1, i0, i1;
  int32_t* err;

  __device__ void init(const int32_t* row_ptr, const int32_t* cols, int64_t b, int64_t nnz, int32_t m, int32_t* e) {
    err = e;
    if constexpr (BLK == 128) {
      i0 = m;
      i1 = -1;
    } else {
      i0 = 2 * m;
      i1 = (2 * m + 1 < b) ? 2 * m + 1 : -1;
    }
    auto row = [&](int32_t i, const int32_t*& c, int32_t& cnt) {
      if (i < 0) {
        c = cols;
        cnt = 0;
        return;
      }
      int32_t a = row_ptr[i], z = row_ptr[i + 1];
      if (a < 0 || z < a || z > nnz) {
        record_error(err, GUARD_BAD_CSR);
        a = z = 0;
      }
      c = cols + a;
      cnt = z - a;
    };
    row(i0, c0, n0);
    row(i1, c1, n1);
    p0 = p1 = 0;
    last0 = last1 = -1;
  }
  // next valid entry of a row (in [0, i], strictly ascending), or INT_MAX
  __device__ int32_t peek(const int32_t* c, int32_t n, int32_t& p, int32_t& last, int32_t i) {
    while (p < n) {
      const int32_t v = c[p];
      if (v >= 0 && v <= i && v > last) return v;
      record_error(err, GUARD_BAD_CSR);
      ++p;
    }
    return 0x7fffffff;
  }
  // next union block and its 2-bit mask (bit 0: row i0, bit 1: row i1); false when done
  __device__ bool next_block(int32_t& blk, int32_t& msk) {
    const int32_t a = peek(c0, n0, p0, last0, i0);
    const int32_t z = (i1 >= 0) ? peek(c1, n1, p1, last1, i1) : 0x7fffffff;
    if (a == 0x7fffffff && z == 0x7fffffff) return false;
    blk = min(a, z);
    msk = 0;
    if (a == blk) {
      msk |= 1;
      last0 = a;
      ++p0;
    }
    if (z == blk) {
      msk |= 2;
      last1 = z;
      ++p1;
    }
    return true;
  }
  // next key tile; returns false when the item has no tile left
  __device__ bool next_tile(TileMeta& t) {
    int32_t b0, m0;
    if (!next_block(b0, m0)) return false;
    t.u0 = b0;
    if constexpr (BLK == 128) {
      t.u1 = b0;
      t.mask = 1;
    } else {
      int32_t b1, m1;
      if (next_block(b1, m1)) {
        t.u1 = b1;
        t.mask = m0 | (m1 << 2);
      } else {
        t.u1 = b0;
        t.mask = m0;
      }
    }
    return true;
  }
};

template <int D, int BLK>
__global__ void __launch_bounds__(kTcThreads, 1) attn_tc_kernel(
    const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
    const __grid_constant__ CUtensorMap tmv, int64_t n, int32_t hq, int32_t group, const int32_t* __restrict__ row_ptr,
    const int32_t* __restrict__ col_idx, int64_t nnz, __nv_bfloat16* __restrict__ o, float qscale, int32_t* err) {
  using L = Smem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars* bs = reinterpret_cast<Bars*>(smem + L::bars);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t b = ceil_div64(n, BLK);
  const int32_t ntiles = static_cast<int32_t>(ceil_div64(n, kTileM));
  const int64_t items = static_cast<int64_t>(ntiles) * hq;

  if (threadIdx.x == 0) {
    mbar_init(&bs->q_full, 1);
    mbar_init(&bs->q_empty, 1);
    mbar_init(&bs->o_empty, 128);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bs->kv_full[s], 1);
      mbar_init(&bs->kv_empty[s], 1);
      mbar_init(&bs->s_full[s], 1);
      mbar_init(&bs->s_empty[s], 128);
      mbar_init(&bs->p_full[s], 128);
      mbar_init(&bs->pv_done[s], 1);
    }
    bs->abort = 0;
    mbar_fence_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(smem_u32(&bs->tmem_base))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bs->tmem_base;

  auto item_of = [&](int64_t t, int32_t& h, int32_t& m) {
    m = ntiles - 1 - static_cast<int32_t>(t / hq);  // longest rows first
    h = static_cast<int32_t>(t % hq);
  };

  if (warp == 0) {
    // ------------------------------------------------------------- producer --
    if (lane == 0) {
      uint32_t kv_it = 0, item_cnt = 0;
      for (int64_t t = blockIdx.x; t < items && !bs->abort; t += gridDim.x, ++item_cnt) {
        int32_t h, m;
        item_of(t, h, m);
        const int32_t g = h / group;
        if (!wait_bar(&bs->q_empty, (item_cnt & 1) ^ 1, bs, err)) break;
        mbar_arrive_expect_tx(&bs->q_full, L::kQ);
#pragma unroll
        for (int a = 0; a < D / 64; ++a)
          tma_load_3d(smem + L::q + a * (kTileM * 128), &tmq, a * 64, m * kTileM, h, &bs->q_full);
        TileWalker<BLK> wk;
        wk.init(row_ptr + static_cast<int64_t>(h) * (b + 1), col_idx + static_cast<int64_t>(h) * nnz, b, nnz, m, err);
        TileMeta cur, nxt;
        bool have = wk.next_tile(cur);
        if (!have) {  // a corrupt CSR row: keep the pipeline shape with one fully masked tile
          cur.u0 = cur.u1 = 0;
          cur.mask = 0;
        }
        bool done = false;
        while (!done) {
          const bool more = have && wk.next_tile(nxt);
          cur.last = more ? 0 : 1;
          const int st = kv_it & 1;
          if (!wait_bar(&bs->kv_empty[st], ((kv_it >> 1) & 1) ^ 1, bs, err)) {
            done = true;
            break;
          }
          bs->meta[st] = cur;
          mbar_arrive_expect_tx(&bs->kv_full[st], 2 * L::kK);
          uint8_t* ks = smem + L::k0 + st * L::kK;
          uint8_t* vs = smem + L::v0 + st * L::kK;
#pragma unroll
          for (int a = 0; a < D / 64; ++a) {
            if constexpr (BLK == 128) {
              tma_load_3d(ks + a * (kTileN * 128), &tmk, a * 64, cur.u0 * 128, g, &bs->kv_full[st]);
              tma_load_3d(vs + a * (kTileN * 128), &tmv, a * 64, cur.u0 * 128, g, &bs->kv_full[st]);
            } else {
              tma_load_3d(ks + a * (kTileN * 128), &tmk, a * 64, cur.u0 * 64, g, &bs->kv_full[st]);
              tma_load_3d(ks + a * (kTileN * 128) + 64 * 128, &tmk, a * 64, cur.u1 * 64, g, &bs->kv_full[st]);
              tma_load_3d(vs + a * (kTileN * 128), &tmv, a * 64, cur.u0 * 64, g, &bs->kv_full[st]);
              tma_load_3d(vs + a * (kTileN * 128) + 64 * 128, &tmv, a * 64, cur.u1 * 64, g, &bs->kv_full[st]);
            }
          }
          ++kv_it;
          if (!more) done = true;
          cur = nxt;
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer --
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16(kTileN, false);
      constexpr uint32_t idPV = idesc_bf16(D, true);
      const uint32_t sq = smem_u32(smem + L::q);
      uint32_t kv_it = 0, gt = 0, item_cnt = 0;
      bool ok = true;
      for (int64_t t = blockIdx.x; ok && t < items; t += gridDim.x, ++item_cnt) {
        if (!(ok = wait_bar(&bs->q_full, item_cnt & 1, bs, err))) break;
        int32_t prev_st = -1;
        uint32_t prev_gt = 0;
        bool first_pv = true;
        auto issue_pv = [&](int st, uint32_t tile) -> bool {
          const int pb = tile & 1;
          if (!wait_bar(&bs->p_full[pb], (tile >> 1) & 1, bs, err)) return false;
          if (first_pv && !wait_bar(&bs->o_empty, (item_cnt & 1) ^ 1, bs, err)) return false;
          tc_fence_after();
          const uint32_t sp = smem_u32(smem + L::p0 + pb * L::kP);
          const uint32_t sv = smem_u32(smem + L::v0 + st * L::kK);
#pragma unroll
          for (int kk = 0; kk < kTileN / 16; ++kk) {
            const uint64_t ad = sw128_desc(sp + (kk >> 2) * (kTileM * 128) + (kk & 3) * 32, 16, 1024);
            const uint64_t bd = sw128_desc(sv + kk * 16 * 128, kTileN * 128, 1024);
            tc_mma(tmem + 256, ad, bd, idPV, (first_pv && kk == 0) ? 0u : 1u);
          }
          tc_commit(&bs->pv_done[pb]);
          tc_commit(&bs->kv_empty[st]);
          first_pv = false;
          return true;
        };
        while (true) {
          const int st = kv_it & 1;
          if (!(ok = wait_bar(&bs->kv_full[st], (kv_it >> 1) & 1, bs, err))) break;
          const bool last = bs->meta[st].last != 0;
          const int sb = gt & 1;
          if (!(ok = wait_bar(&bs->s_empty[sb], ((gt >> 1) & 1) ^ 1, bs, err))) break;
          tc_fence_after();
          const uint32_t sk = smem_u32(smem + L::k0 + st * L::kK);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * (kTileM * 128) + (kk & 3) * 32;
            const uint32_t koff = (kk >> 2) * (kTileN * 128) + (kk & 3) * 32;
            tc_mma(tmem + sb * kTileN, sw128_desc(sq + off, 16, 1024), sw128_desc(sk + koff, 16, 1024), idS,
                   kk > 0 ? 1u : 0u);
          }
          tc_commit(&bs->s_full[sb]);
          if (last) tc_commit(&bs->q_empty);
          if (prev_st >= 0 && !(ok = issue_pv(prev_st, prev_gt))) break;
          prev_st = st;
          prev_gt = gt;
          ++kv_it;
          ++gt;
          if (last) {
            ok = issue_pv(prev_st, prev_gt);
            break;
          }
        }
      }
    }
  } else {
    // -------------------------------------------------------------- softmax --
    const int q4 = warp & 3;        // TMEM lane quarter of this warp
    const int r = q4 * 32 + lane;   // query row of the tile
    const uint32_t trow = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    uint32_t kv_it = 0, gt = 0;
    bool ok = true;
    for (int64_t t = blockIdx.x; ok && t < items; t += gridDim.x) {
      int32_t h, m;
      item_of(t, h, m);
      const int64_t tok = static_cast<int64_t>(m) * kTileM + r;
      const int qh = r >> 6;  // query half (B = 64)
      float m_used = -INFINITY, l = 0.f;
      bool first_tile = true;
      while (true) {
        const int st = kv_it & 1;
        if (!(ok = warp_wait(&bs->kv_full[st], (kv_it >> 1) & 1, bs, err))) break;
        const TileMeta tm = bs->meta[st];
        const int sb = gt & 1;
        if (!(ok = warp_wait(&bs->s_full[sb], (gt >> 1) & 1, bs, err))) break;
        tc_fence_after();
        float s[kTileN];
#pragma unroll
        for (int c = 0; c < kTileN / 32; ++c) {
          float v[32];
          tmem_ld32(trow + sb * kTileN + c * 32, v);
#pragma unroll
          for (int i = 0; i < 32; ++i) s[c * 32 + i] = v[i];
        }
        tc_fence_before();
        mbar_arrive(&bs->s_empty[sb]);
        // masks: 0 = none, 1 = all, 2 = causal (key offset <= query offset)
        int mode[2];
        int limit[2];
        if constexpr (BLK == 128) {
          mode[0] = mode[1] = (tm.u0 < m) ? 1 : 2;
          limit[0] = r;
          limit[1] = r - 64;
        } else {
          const int qi = 2 * m + qh;
#pragma unroll
          for (int kh = 0; kh < 2; ++kh) {
            const int kb = kh ? tm.u1 : tm.u0;
            const bool sel = (tm.mask >> (2 * kh + qh)) & 1;
            mode[kh] = !sel ? 0 : (kb < qi ? 1 : (kb == qi ? 2 : 0));
            limit[kh] = r & 63;
          }
        }
        float mx = -INFINITY;
#pragma unroll
        for (int c = 0; c < kTileN; ++c) {
          const int kh = c >> 6;
          const int cc = (BLK == 128) ? c : (c & 63);
          const bool valid = mode[kh] == 1 || (mode[kh] == 2 && cc <= ((BLK == 128) ? r : limit[kh]));
          s[c] = valid ? s[c] : -INFINITY;
          mx = fmaxf(mx, s[c]);
        }
        const float m_new = mx * qscale;
        const bool need = mx != -INFINITY && (m_used == -INFINITY || m_new > m_used + kRescaleLog2);
        const float alpha = need ? fast_exp2(m_used - m_new) : 1.f;  // 0 when m_used = -inf
        if (!first_tile && __any_sync(0xffffffffu, need)) {
          // O holds earlier tiles at the old reference: wait for them, then the
          // whole warp rescales its rows (alpha = 1 for rows that keep theirs)
          if (!(ok = warp_wait(&bs->pv_done[(gt - 1) & 1], ((gt - 1) >> 1) & 1, bs, err))) break;
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            float v[32];
            tmem_ld32(trow + 256 + c * 32, v);
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] *= alpha;
            tmem_st32(trow + 256 + c * 32, v);
          }
          tmem_wait_st();
        }
        if (need) {
          l *= alpha;
          m_used = m_new;
        }
        // P = 2^(s * qscale - m_used); masked entries and an unset reference give 0
        float psum = 0.f;
        uint32_t pk[kTileN / 2];
#pragma unroll
        for (int c = 0; c < kTileN; c += 2) {
          const float p0 = (m_used == -INFINITY) ? 0.f : fast_exp2(fmaf(s[c], qscale, -m_used));
          const float p1 = (m_used == -INFINITY) ? 0.f : fast_exp2(fmaf(s[c + 1], qscale, -m_used));
          psum += p0 + p1;
          pk[c >> 1] = pack_bf16x2(p0, p1);
        }
        l += psum;
        // the P buffer was last read by the PV of tile gt - 2
        if (gt >= 2 && !(ok = warp_wait(&bs->pv_done[sb], ((gt - 2) >> 1) & 1, bs, err))) break;
        uint8_t* prow = smem + L::p0 + sb * L::kP + r * 128;
#pragma unroll
        for (int ch = 0; ch < kTileN / 8; ++ch) {
          const int atom = ch >> 3, cc = ch & 7;
          uint4 v = make_uint4(pk[ch * 4], pk[ch * 4 + 1], pk[ch * 4 + 2], pk[ch * 4 + 3]);
          *reinterpret_cast<uint4*>(prow + atom * (kTileM * 128) + ((cc ^ (r & 7)) << 4)) = v;
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        tc_fence_before();
        mbar_arrive(&bs->p_full[sb]);
        first_tile = false;
        ++kv_it;
        ++gt;
        if (tm.last) break;
      }
      if (!ok) break;
      // epilogue: O / l for this row, once every PV of the item has completed
      if (!(ok = warp_wait(&bs->pv_done[(gt - 1) & 1], ((gt - 1) >> 1) & 1, bs, err))) break;
      tc_fence_after();
      const float inv = (l > 0.f) ? 1.f / l : 0.f;
      __nv_bfloat16* orow = o + (static_cast<int64_t>(h) * n + tok) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        float v[32];
        tmem_ld32(trow + 256 + c * 32, v);
        if (tok < n) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 w = make_uint4(pack_bf16x2(v[q * 8 + 0] * inv, v[q * 8 + 1] * inv),
                                 pack_bf16x2(v[q * 8 + 2] * inv, v[q * 8 + 3] * inv),
                                 pack_bf16x2(v[q * 8 + 4] * inv, v[q * 8 + 5] * inv),
                                 pack_bf16x2(v[q * 8 + 6] * inv, v[q * 8 + 7] * inv));
            *reinterpret_cast<uint4*>(orow + c * 32 + q * 8) = w;
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&bs->o_empty);
    }
  }
  // teardown: the softmax warps waited for the last PV of their last item, and
  // MMAs complete in issue order, so no MMA is in flight past this barrier
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
  }
}

// ---- host side -------------------------------------------------------------------

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// [heads][rows][D] bf16 as a 3-D tensor map with a {64, box_rows, 1} box, 128-byte swizzle.
bool make_map(CUtensorMap* map, const void* base, int64_t rows, int32_t heads, int D, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows),
                              static_cast<cuuint64_t>(heads)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(rows) * D * 2};
  const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int BLK>
cudaError_t launch_tc(const sws_handle* h, const void* q, const void* k, const void* v, int64_t n, int32_t hq,
                      int32_t hkv, const int32_t* row_ptr, const int32_t* col_idx, void* o, cudaStream_t st) {
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, q, n, hq, D, kTileM) || !make_map(&mk, k, n, hkv, D, BLK == 128 ? 128 : 64) ||
      !make_map(&mv, v, n, hkv, D, BLK == 128 ? 128 : 64))
    return cudaErrorInvalidValue;
  const size_t smem = Smem<D>::total + 1024;
  auto kern = attn_tc_kernel<D, BLK>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int64_t b = ceil_div64(n, BLK);
  int64_t nnz = 0;
  for (int64_t i = 0; i < b; ++i) nnz += tau_of_row(i, h->cfg.density_num, h->cfg.density_den);
  const int64_t items = ceil_div64(n, kTileM) * hq;
  const int grid = static_cast<int>(std::min<int64_t>(items, h->num_sms));
  const float qscale = static_cast<float>(1.4426950408889634 / sqrt(static_cast<double>(D)));
  kern<<<grid, kTcThreads, smem, st>>>(mq, mk, mv, n, hq, hq / hkv, row_ptr, col_idx, nnz,
                                       static_cast<__nv_bfloat16*>(o), qscale, h->err);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace

size_t attn_prefill_tc_smem_bytes(int d) { return (d == 128 ? Smem<128>::total : Smem<64>::total) + 1024; }

cudaError_t launch_attn_prefill_tc(const sws_handle* h, const void* q, const void* k, const void* v, int64_t n,
                                   int32_t hq, int32_t hkv, const int32_t* row_ptr, const int32_t* col_idx, void* o,
                                   cudaStream_t st) {
  const int d = h->cfg.head_dim, B = h->cfg.block_size;
  if (d == 128) {
    return B == 128 ? launch_tc<128, 128>(h, q, k, v, n, hq, hkv, row_ptr, col_idx, o, st)
                    : launch_tc<128, 64>(h, q, k, v, n, hq, hkv, row_ptr, col_idx, o, st);
  }
  return B == 128 ? launch_tc<64, 128>(h, q, k, v, n, hq, hkv, row_ptr, col_idx, o, st)
                  : launch_tc<64, 64>(h, q, k, v, n, hq, hkv, row_ptr, col_idx, o, st);
}

}  // namespace sws
