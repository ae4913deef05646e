// sw_sparse_attn_prefill on the 5th-generation tensor cores (bf16 in, fp32 accumulate).
//
// "Scout Before You Attend" §4/§5: exact softmax attention on the original
// Q, K, V restricted to the key blocks selected for each query block (query
// token t sees key token u of a selected block iff u <= t).
//
// One persistent CTA per SM walks (head, 256-row query slab) work items,
// longest first. A slab is two 128-row query tiles that share one stream of
// 128-key tiles: the merged CSR rows of its query blocks (4 blocks of 64 or 2
// of 128; adjacent query blocks select almost the same key blocks), each key
// tile carrying a selection bit per (key block, query block) pair.
//
// Warp roles (352 threads):
//   warp 0    TMA producer: both Q tiles once per item, then K tiles into a
//             3-stage ring and V tiles into a 2-stage ring (3-D tensor maps,
//             128-byte swizzle, zero fill past n); the score products run ahead
//             of the PV products, so K is needed before V;
//   warp 1    owns the 512 TMEM columns and issues the score products
//             S_w = Q_w K^T of the two query tiles w, S_0(g), S_1(g), S_0(g+1),
//             ..., into the one score buffer the tiles share; each waits until
//             the softmax group of the previous product has copied the buffer
//             to registers;
//   warp 10   issues O_w += P_w V with P_w read from the tile's own TMEM
//             columns, once the softmax group has written it. With two issuing
//             threads the tensor cores are fed while either one waits, and no
//             product ever waits for another product to finish;
//   warps 2-5 and 6-9: one softmax warpgroup per query tile, one query row per
//             thread (TMEM lane = row). A row keeps a running max that only
//             moves when it grows by more than 2^8 (then its row of O in TMEM is
//             rescaled); P = 2^(s - m) goes to the group's P columns as bf16 once
//             its previous PV has read them; the group finally writes O / l.
// Every wait is bounded; a timeout records a guard code and all roles leave.
//
// Packed sequences (kVar): one launch over several sequences laid end to end
// along the token axis of Q, K, V and O. A table of (sequence, slab) entries,
// longest slabs first across all sequences, replaces the slab index, and each
// sequence brings its own token offset, length and CSR. Keys past a
// sequence's end are never unmasked (a selected block before the query's own
// is complete, and the diagonal block is causal), and rows past its end are
// not written, so sequences never see each other. The pipeline itself (the
// barriers, the roles) does not change: the MMA issuers never look at an
// item's identity.
#include <cuda.h>

#include <algorithm>
#include <vector>

#include "sws_common.cuh"

namespace sws {
namespace {

constexpr int kTcThreads = 352;  // 11 warps
constexpr int kTileM = 128;   // query rows per tile (two tiles per item)
constexpr int kTileN = 128;   // keys per S tile
constexpr int kGroup = 128;   // threads per softmax warpgroup
constexpr int kKStages = 3, kVStages = 2;
constexpr int kPvWarp = 10;   // issues the PV products
// arrivals per softmax-group barrier phase: one per warp, after __syncwarp
constexpr int kArrivals = kGroup / 32;

__device__ __forceinline__ void group_arrive(uint64_t* bar) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}
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

__device__ __forceinline__ uint32_t pack_p(float lo, float hi) { return pack_bf16x2(lo, hi); }

// Two fp32 lanes in one 64-bit register for the packed fp32x2 instructions.
__device__ __forceinline__ uint64_t f2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_split(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// 32 columns of this thread's lane into r[]; the registers become valid only
// after tmem_wait_ld4 below, which names them as operands so that no use can
// move above it.
__device__ __forceinline__ void tmem_ld32_nw(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];" : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]) : "r"(taddr) : "memory");
}
__device__ __forceinline__ void tmem_wait_ld4(uint32_t (&a)[32], uint32_t (&b)[32], uint32_t (&c)[32], uint32_t (&d)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;" : "+r"(a[0]), "+r"(b[0]), "+r"(c[0]), "+r"(d[0]), "+r"(a[1]), "+r"(b[1]), "+r"(c[1]), "+r"(d[1]), "+r"(a[2]), "+r"(b[2]), "+r"(c[2]), "+r"(d[2]), "+r"(a[3]), "+r"(b[3]), "+r"(c[3]), "+r"(d[3]), "+r"(a[4]), "+r"(b[4]), "+r"(c[4]), "+r"(d[4]), "+r"(a[5]), "+r"(b[5]), "+r"(c[5]), "+r"(d[5]), "+r"(a[6]), "+r"(b[6]), "+r"(c[6]), "+r"(d[6]), "+r"(a[7]), "+r"(b[7]), "+r"(c[7]), "+r"(d[7]), "+r"(a[8]), "+r"(b[8]), "+r"(c[8]), "+r"(d[8]), "+r"(a[9]), "+r"(b[9]), "+r"(c[9]), "+r"(d[9]), "+r"(a[10]), "+r"(b[10]), "+r"(c[10]), "+r"(d[10]), "+r"(a[11]), "+r"(b[11]), "+r"(c[11]), "+r"(d[11]), "+r"(a[12]), "+r"(b[12]), "+r"(c[12]), "+r"(d[12]), "+r"(a[13]), "+r"(b[13]), "+r"(c[13]), "+r"(d[13]), "+r"(a[14]), "+r"(b[14]), "+r"(c[14]), "+r"(d[14]), "+r"(a[15]), "+r"(b[15]), "+r"(c[15]), "+r"(d[15]), "+r"(a[16]), "+r"(b[16]), "+r"(c[16]), "+r"(d[16]), "+r"(a[17]), "+r"(b[17]), "+r"(c[17]), "+r"(d[17]), "+r"(a[18]), "+r"(b[18]), "+r"(c[18]), "+r"(d[18]), "+r"(a[19]), "+r"(b[19]), "+r"(c[19]), "+r"(d[19]), "+r"(a[20]), "+r"(b[20]), "+r"(c[20]), "+r"(d[20]), "+r"(a[21]), "+r"(b[21]), "+r"(c[21]), "+r"(d[21]), "+r"(a[22]), "+r"(b[22]), "+r"(c[22]), "+r"(d[22]), "+r"(a[23]), "+r"(b[23]), "+r"(c[23]), "+r"(d[23]), "+r"(a[24]), "+r"(b[24]), "+r"(c[24]), "+r"(d[24]), "+r"(a[25]), "+r"(b[25]), "+r"(c[25]), "+r"(d[25]), "+r"(a[26]), "+r"(b[26]), "+r"(c[26]), "+r"(d[26]), "+r"(a[27]), "+r"(b[27]), "+r"(c[27]), "+r"(d[27]), "+r"(a[28]), "+r"(b[28]), "+r"(c[28]), "+r"(d[28]), "+r"(a[29]), "+r"(b[29]), "+r"(c[29]), "+r"(d[29]), "+r"(a[30]), "+r"(b[30]), "+r"(c[30]), "+r"(d[30]), "+r"(a[31]), "+r"(b[31]), "+r"(c[31]), "+r"(d[31]) :: "memory");
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

__device__ __forceinline__ void tc_mma_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
      "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}


// Stores 16 packed words into 16 consecutive columns of this thread's lane.
__device__ __forceinline__ void tmem_st16u(uint32_t taddr, const uint32_t* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
          taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}

// ---- shared state ----------------------------------------------------------------

// One sequence of a packed launch: rows tok0 .. tok0 + n - 1 of the packed
// tensors; per head its CSR has b + 1 offsets (row_ptr + h (b + 1)) and nnz
// columns (col_idx + h nnz).
struct SeqDesc {
  const int32_t* row_ptr;
  const int32_t* col_idx;
  int64_t nnz, n, tok0, b;
};

// What a role needs of one work item.
struct ItemCtx {
  int32_t h, p;  // query head, 256-row slab of the sequence
  int64_t tok0, n, b, nnz;
  const int32_t* rp;  // the head's CSR
  const int32_t* ci;
};

struct TileMeta {
  int32_t u0, u1;  // key blocks of the two 64-key halves (B = 64), or the key block twice (B = 128)
  int32_t mask;    // bit (key_block_slot * QB + query_block_slot): that query block selected that key block
  int32_t last;    // last key tile of the item
};

struct Bars {
  uint64_t q_full, q_empty;
  uint64_t k_full[kKStages], k_empty[kKStages], v_full[kVStages], v_empty[kVStages];
  uint64_t s_full[2], s_free[2], p_full[2], pv_done[2], o_empty[2];  // per query tile
  TileMeta meta[kKStages];  // per K stage
  uint32_t tmem_base;
  volatile int32_t abort;
};

template <int D>
struct Smem {
  static constexpr uint32_t kQ = kTileM * D * 2;  // one query tile
  static constexpr uint32_t kK = kTileN * D * 2;
  static constexpr uint32_t q = 0;                // two query tiles
  static constexpr uint32_t k0 = q + 2 * kQ;
  static constexpr uint32_t v0 = k0 + kKStages * kK;
  static constexpr uint32_t bars = v0 + kVStages * kK;
  static constexpr uint32_t total = bars + sizeof(Bars);
};

// TMEM columns: the shared score buffer at 0, P_w (bf16 pairs) at 128 + 64 w,
// O_w at 256 + 128 w.
constexpr uint32_t kColS = 0;
__host__ __device__ constexpr uint32_t tcol_p(int w) { return 128u + 64u * w; }
__host__ __device__ constexpr uint32_t tcol_o(int w) { return 256u + 128u * w; }

// Bounded wait (wall time) that also gives up as soon as another role has aborted.
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, Bars* bs, int32_t* err) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 15) == 0) {
      if (bs->abort) return false;
      if (global_ns() - t0 > kWaitNs) break;
    }
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

// Walks the key tiles of one item: the merge of the CSR rows of its QB query
// blocks; B = 128: one key block per tile, B = 64: two union blocks per tile.
template <int BLK>
struct TileWalker {
  static constexpr int QB = 256 / BLK;
  const int32_t* c[QB];
  int32_t cnt[QB], pos[QB], last[QB], row[QB];
  int32_t* err;

  __device__ void init(const int32_t* row_ptr, const int32_t* cols, int64_t b, int64_t nnz, int32_t p, int32_t* e) {
    err = e;
#pragma unroll
    for (int q = 0; q < QB; ++q) {
      const int64_t i = static_cast<int64_t>(p) * QB + q;
      row[q] = static_cast<int32_t>(i);
      pos[q] = 0;
      last[q] = -1;
      c[q] = cols;
      cnt[q] = 0;
      if (i < b) {
        int32_t a = row_ptr[i], z = row_ptr[i + 1];
        if (a < 0 || z < a || z > nnz) {
          record_error(err, GUARD_BAD_CSR);
          a = z = 0;
        }
        c[q] = cols + a;
        cnt[q] = z - a;
      }
    }
  }
  // next valid entry of row q (in [0, i], strictly ascending), or INT_MAX
  __device__ int32_t peek(int q) {
    while (pos[q] < cnt[q]) {
      const int32_t v = c[q][pos[q]];
      if (v >= 0 && v <= row[q] && v > last[q]) return v;
      record_error(err, GUARD_BAD_CSR);
      ++pos[q];
    }
    return 0x7fffffff;
  }
  // next union block and its QB-bit mask; false when done
  __device__ bool next_block(int32_t& blk, int32_t& msk) {
    int32_t h[QB];
    int32_t mn = 0x7fffffff;
#pragma unroll
    for (int q = 0; q < QB; ++q) {
      h[q] = peek(q);
      mn = min(mn, h[q]);
    }
    if (mn == 0x7fffffff) return false;
    blk = mn;
    msk = 0;
#pragma unroll
    for (int q = 0; q < QB; ++q)
      if (h[q] == mn) {
        msk |= 1 << q;
        last[q] = mn;
        ++pos[q];
      }
    return true;
  }
  __device__ bool next_tile(TileMeta& t) {
    int32_t b0, m0;
    if (!next_block(b0, m0)) return false;
    t.u0 = b0;
    if constexpr (BLK == 128) {
      t.u1 = b0;
      t.mask = m0;
    } else {
      int32_t b1, m1;
      if (next_block(b1, m1)) {
        t.u1 = b1;
        t.mask = m0 | (m1 << QB);
      } else {
        t.u1 = b0;
        t.mask = m0;
      }
    }
    return true;
  }
};

template <int D, int BLK, bool kVar>
__global__ void __launch_bounds__(kTcThreads, 1) attn_tc_kernel(
    const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
    const __grid_constant__ CUtensorMap tmv, int64_t n, int32_t hq, int32_t group, const int32_t* __restrict__ row_ptr,
    const int32_t* __restrict__ col_idx, int64_t nnz, __nv_bfloat16* __restrict__ o, HeadTok os, float qscale,
    const SeqDesc* __restrict__ seqs, const int2* __restrict__ ents, int32_t nent, int32_t* err) {
  grid_dependency_wait();
  allow_dependents();
  using L = Smem<D>;
  constexpr int QB = 256 / BLK;  // query blocks per item
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars* bs = reinterpret_cast<Bars*>(smem + L::bars);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t b = ceil_div64(n, BLK);
  const int32_t nslab = static_cast<int32_t>(ceil_div64(n, 2 * kTileM));
  const int64_t items = static_cast<int64_t>(kVar ? nent : nslab) * hq;

  if (threadIdx.x == 0) {
    mbar_init(&bs->q_full, 1);
    mbar_init(&bs->q_empty, 1);
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(&bs->k_full[s], 1);
      mbar_init(&bs->k_empty[s], 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(&bs->v_full[s], 1);
      mbar_init(&bs->v_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bs->s_full[s], 1);
      mbar_init(&bs->s_free[s], kArrivals);
      mbar_init(&bs->p_full[s], kArrivals);
      mbar_init(&bs->pv_done[s], 1);
      mbar_init(&bs->o_empty[s], kArrivals);
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

  auto item_of = [&](int64_t t) {
    ItemCtx c;
    c.h = static_cast<int32_t>(t % hq);
    if constexpr (kVar) {
      const int2 e = ents[t / hq];  // sorted longest slab first on the host
      const SeqDesc* sd = seqs + e.x;
      c.p = e.y;
      c.tok0 = sd->tok0;
      c.n = sd->n;
      c.b = sd->b;
      c.nnz = sd->nnz;
      c.rp = sd->row_ptr + static_cast<int64_t>(c.h) * (c.b + 1);
      c.ci = sd->col_idx + static_cast<int64_t>(c.h) * c.nnz;
    } else {
      c.p = nslab - 1 - static_cast<int32_t>(t / hq);  // longest rows first
      c.tok0 = 0;
      c.n = n;
      c.b = b;
      c.nnz = nnz;
      c.rp = row_ptr + static_cast<int64_t>(c.h) * (b + 1);
      c.ci = col_idx + static_cast<int64_t>(c.h) * nnz;
    }
    return c;
  };

  if (warp == 0) {
    // ------------------------------------------------------------- producer --
    if (lane == 0) {
      uint32_t kv_it = 0, item_cnt = 0;
      for (int64_t t = blockIdx.x; t < items && !bs->abort; t += gridDim.x, ++item_cnt) {
        const ItemCtx it = item_of(t);
        const int32_t h = it.h, p = it.p;
        const int32_t tok0 = static_cast<int32_t>(it.tok0);  // the packed token count fits in 32 bits
        const int32_t g = h / group;
        if (!wait_bar(&bs->q_empty, (item_cnt & 1) ^ 1, bs, err)) break;
        mbar_arrive_expect_tx(&bs->q_full, 2 * L::kQ);
#pragma unroll
        for (int w = 0; w < 2; ++w)
#pragma unroll
          for (int a = 0; a < D / 64; ++a)
            tma_load_3d(smem + L::q + w * L::kQ + a * (kTileM * 128), &tmq, a * 64,
                        tok0 + p * 2 * kTileM + w * kTileM, h, &bs->q_full);
        TileWalker<BLK> wk;
        wk.init(it.rp, it.ci, it.b, it.nnz, p, err);
        TileMeta cur, nxt;
        bool have = wk.next_tile(cur);
        if (!have) {  // a corrupt CSR: keep the pipeline shape with one fully masked tile
          cur.u0 = cur.u1 = 0;
          cur.mask = 0;
        }
        bool done = false;
        while (!done) {
          const bool more = have && wk.next_tile(nxt);
          cur.last = more ? 0 : 1;
          const int sk = kv_it % kKStages, sv = kv_it % kVStages;
          if (!wait_bar(&bs->k_empty[sk], ((kv_it / kKStages) & 1) ^ 1, bs, err)) break;
          bs->meta[sk] = cur;
          mbar_arrive_expect_tx(&bs->k_full[sk], L::kK);
          uint8_t* ks = smem + L::k0 + sk * L::kK;
#pragma unroll
          for (int a = 0; a < D / 64; ++a) {
            if constexpr (BLK == 128) {
              tma_load_3d(ks + a * (kTileN * 128), &tmk, a * 64, tok0 + cur.u0 * 128, g, &bs->k_full[sk]);
            } else {
              tma_load_3d(ks + a * (kTileN * 128), &tmk, a * 64, tok0 + cur.u0 * 64, g, &bs->k_full[sk]);
              tma_load_3d(ks + a * (kTileN * 128) + 64 * 128, &tmk, a * 64, tok0 + cur.u1 * 64, g, &bs->k_full[sk]);
            }
          }
          if (!wait_bar(&bs->v_empty[sv], ((kv_it / kVStages) & 1) ^ 1, bs, err)) break;
          mbar_arrive_expect_tx(&bs->v_full[sv], L::kK);
          uint8_t* vs = smem + L::v0 + sv * L::kK;
#pragma unroll
          for (int a = 0; a < D / 64; ++a) {
            if constexpr (BLK == 128) {
              tma_load_3d(vs + a * (kTileN * 128), &tmv, a * 64, tok0 + cur.u0 * 128, g, &bs->v_full[sv]);
            } else {
              tma_load_3d(vs + a * (kTileN * 128), &tmv, a * 64, tok0 + cur.u0 * 64, g, &bs->v_full[sv]);
              tma_load_3d(vs + a * (kTileN * 128) + 64 * 128, &tmv, a * 64, tok0 + cur.u1 * 64, g, &bs->v_full[sv]);
            }
          }
          ++kv_it;
          if (!more) done = true;
          cur = nxt;
        }
      }
    }
  } else if (warp == 1 || warp == kPvWarp) {
    // ------------------------------------------------------------ MMA issuers --
    // Two threads feed the tensor cores, so that neither stream's waits leave
    // them idle: warp 1 issues the score products S_0(g), S_1(g), S_0(g+1), ...
    // into the one score buffer, each once the softmax group of the previous
    // one has copied the buffer to registers (s_free); warp kPvWarp issues
    // PV_0(g), PV_1(g), PV_0(g+1), ..., each once its P is in TMEM (p_full) and,
    // on an item's first tile, once the previous item's epilogue has read O_w
    // (o_empty). Each thread commits the barriers of its own products.
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16(kTileN, false);
      constexpr uint32_t idPV = idesc_bf16(D, true);
      const bool s_stream = warp == 1;
      uint32_t g = 0, item_g = 0;
      bool ok = true;
      for (int64_t t = blockIdx.x; ok && t < items; t += gridDim.x, ++item_g) {
        if (s_stream && !(ok = wait_bar(&bs->q_full, item_g & 1, bs, err))) break;
        bool first = true;
        while (true) {
          const int sk = g % kKStages;
          if (!(ok = wait_bar(&bs->k_full[sk], (g / kKStages) & 1, bs, err))) break;
          const bool last = bs->meta[sk].last != 0;
          if (s_stream) {
            const uint32_t sq0 = smem_u32(smem + L::q), sq1 = smem_u32(smem + L::q + L::kQ);
            const uint32_t skk = smem_u32(smem + L::k0 + sk * L::kK);
            if (g > 0 && !(ok = wait_bar(&bs->s_free[1], (g - 1) & 1, bs, err))) break;
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off = (kk >> 2) * (kTileM * 128) + (kk & 3) * 32;
              const uint32_t koff = (kk >> 2) * (kTileN * 128) + (kk & 3) * 32;
              tc_mma(tmem + kColS, sw128_desc(sq0 + off, 16, 1024), sw128_desc(skk + koff, 16, 1024), idS,
                     kk > 0 ? 1u : 0u);
            }
            tc_commit(&bs->s_full[0]);
            if (!(ok = wait_bar(&bs->s_free[0], g & 1, bs, err))) break;
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off = (kk >> 2) * (kTileM * 128) + (kk & 3) * 32;
              const uint32_t koff = (kk >> 2) * (kTileN * 128) + (kk & 3) * 32;
              tc_mma(tmem + kColS, sw128_desc(sq1 + off, 16, 1024), sw128_desc(skk + koff, 16, 1024), idS,
                     kk > 0 ? 1u : 0u);
            }
            tc_commit(&bs->s_full[1]);
            if (last) tc_commit(&bs->q_empty);
          } else {
            const uint32_t sv = smem_u32(smem + L::v0 + (g % kVStages) * L::kK);
            if (!(ok = wait_bar(&bs->v_full[g % kVStages], (g / kVStages) & 1, bs, err))) break;
#pragma unroll
            for (int w = 0; w < 2; ++w) {
              if (!(ok = wait_bar(&bs->p_full[w], g & 1, bs, err))) break;
              if (first && !(ok = wait_bar(&bs->o_empty[w], (item_g & 1) ^ 1, bs, err))) break;
              tc_fence_after();
#pragma unroll
              for (int kk = 0; kk < kTileN / 16; ++kk)
                tc_mma_ts(tmem + tcol_o(w), tmem + tcol_p(w) + kk * 8,
                          sw128_desc(sv + kk * 16 * 128, kTileN * 128, 1024), idPV, (first && kk == 0) ? 0u : 1u);
              tc_commit(&bs->pv_done[w]);
            }
            if (!ok) break;
            // K and V of tile g are free (S_1(g) completed before P_1(g) was
            // written); a K stage is released only here, after both softmax
            // groups are done with the tile, because its slot also holds the
            // tile's metadata
            tc_commit(&bs->k_empty[sk]);
            tc_commit(&bs->v_empty[g % kVStages]);
          }
          first = false;
          ++g;
          if (last) break;
        }
      }
    }
  } else if (warp >= 2 && warp < 10) {
    // -------------------------------------------------------------- softmax --
    const int w = (warp - 2) >> 2;          // query tile of this warpgroup
    const int q4 = warp & 3;                // TMEM lane quarter of this warp
    const int r = q4 * 32 + lane;           // query row of the tile
    const uint32_t trow = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    const uint32_t ts = trow + kColS, tp = trow + tcol_p(w), to = trow + tcol_o(w);
    const int qslot = (w * kTileM + r) / BLK;  // query block slot within the item
    uint32_t kv_it = 0, gt = 0, item_cnt = 0;
    bool ok = true;
    for (int64_t t = blockIdx.x; ok && t < items; t += gridDim.x, ++item_cnt) {
      const ItemCtx it = item_of(t);
      const int32_t h = it.h, p = it.p;
      const int64_t tok = static_cast<int64_t>(p) * 2 * kTileM + w * kTileM + r;  // row of the sequence
      const int64_t qi = static_cast<int64_t>(p) * QB + qslot;  // query block of this row
      float m_used = -INFINITY, l = 0.f;
      bool first_tile = true;
      while (true) {
        const int sk = kv_it % kKStages;
        if (!(ok = warp_wait(&bs->k_full[sk], (kv_it / kKStages) & 1, bs, err))) break;
        const TileMeta tm = bs->meta[sk];
        if (!(ok = warp_wait(&bs->s_full[w], gt & 1, bs, err))) break;
        tc_fence_after();
        float s[kTileN];
        {
          uint32_t ra[32], rb[32], rc[32], rd[32];
          tmem_ld32_nw(ts, ra);
          tmem_ld32_nw(ts + 32, rb);
          tmem_ld32_nw(ts + 64, rc);
          tmem_ld32_nw(ts + 96, rd);
          tmem_wait_ld4(ra, rb, rc, rd);
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            s[i] = __uint_as_float(ra[i]);
            s[32 + i] = __uint_as_float(rb[i]);
            s[64 + i] = __uint_as_float(rc[i]);
            s[96 + i] = __uint_as_float(rd[i]);
          }
        }
        // the scores are in registers: the score buffer may take the next product
        tc_fence_before();
        group_arrive(&bs->s_free[w]);
        // masks per key block slot: 0 = none, 1 = all, 2 = causal (key offset <= query offset)
        constexpr int KBS = kTileN / BLK;
        int mode[KBS];
#pragma unroll
        for (int kb = 0; kb < KBS; ++kb) {
          const int64_t ub = kb ? tm.u1 : tm.u0;
          const bool sel = (tm.mask >> (kb * QB + qslot)) & 1;
          mode[kb] = !sel ? 0 : (ub < qi ? 1 : (ub == qi ? 2 : 0));
        }
        const int qoff = r & (BLK - 1);  // offset of the row inside its query block
#pragma unroll
        for (int kb = 0; kb < KBS; ++kb) {
          if (mode[kb] != 1) {
#pragma unroll
            for (int c = 0; c < BLK; ++c)
              s[kb * BLK + c] = (mode[kb] == 2 && c <= qoff) ? s[kb * BLK + c] : -INFINITY;
          }
        }
        float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int c = 0; c < kTileN; c += 8)
#pragma unroll
          for (int u = 0; u < 4; ++u) mx4[u] = max3f(mx4[u], s[c + 2 * u], s[c + 2 * u + 1]);
        const float mx = max3f(mx4[0], mx4[1], fmaxf(mx4[2], mx4[3]));
        const float m_new = mx * qscale;
        const bool need = mx != -INFINITY && (m_used == -INFINITY || m_new > m_used + kRescaleLog2);
        const float alpha = need ? fast_exp2(m_used - m_new) : 1.f;  // 0 when m_used = -inf
        if (need) {
          l *= alpha;
          m_used = m_new;
        }
        // P = 2^(s * qscale - m_used) as packed bf16 pairs, kept in registers
        // until this group's previous PV has read its P columns. Masked scores
        // are -inf and give exactly 0; a row whose reference is still -inf has
        // seen only masked scores, so nm = 0 gives 0 there too. Scale, shift and
        // row sum run on the packed fp32x2 pipe.
        const float nm = m_used != -INFINITY ? -m_used : 0.f;
        const uint64_t sc2 = f2(qscale, qscale), nm2 = f2(nm, nm);
        uint64_t acc2[4] = {0ull, 0ull, 0ull, 0ull};
        uint32_t pk[kTileN / 2];
#pragma unroll
        for (int i = 0; i < kTileN / 2; ++i) {
          const int c = 2 * i;
          float x0, x1;
          f2_split(f2_fma(f2(s[c], s[c + 1]), sc2, nm2), x0, x1);
          const float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
          acc2[i & 3] = f2_add(acc2[i & 3], f2(p0, p1));
          pk[i] = pack_p(p0, p1);
        }
        {
          float a0, a1, b0, b1;
          f2_split(f2_add(acc2[0], acc2[1]), a0, a1);
          f2_split(f2_add(acc2[2], acc2[3]), b0, b1);
          l += (a0 + a1) + (b0 + b1);
        }
        // PV_w(gt-1) has read P_w and written O_w: both may change now. This
        // group waits for every one of its PV completions in turn, so the wait
        // is never more than one phase ahead of the barrier.
        if (gt > 0 && !(ok = warp_wait(&bs->pv_done[w], (gt - 1) & 1, bs, err))) break;
        tc_fence_after();
        if (!first_tile && __any_sync(0xffffffffu, need)) {
          // O_w holds earlier tiles at the old reference: the whole warp
          // rescales its rows (alpha = 1 for rows that keep theirs)
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            float v[32];
            tmem_ld32(to + c * 32, v);
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] *= alpha;
            tmem_st32(to + c * 32, v);
          }
        }
#pragma unroll
        for (int qt = 0; qt < kTileN / 32; ++qt) tmem_st16u(tp + qt * 16, pk + 16 * qt);
        tmem_wait_st();
        tc_fence_before();
        group_arrive(&bs->p_full[w]);
        first_tile = false;
        ++kv_it;
        ++gt;
        if (tm.last) break;
      }
      if (!ok) break;
      // epilogue: O_w / l for this row, once every PV of the item has completed
      if (!(ok = warp_wait(&bs->pv_done[w], (gt - 1) & 1, bs, err))) break;
      tc_fence_after();
      const float inv = (l > 0.f) ? 1.f / l : 0.f;
      __nv_bfloat16* orow = o + h * os.head + (it.tok0 + tok) * os.tok;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        float v[32];
        tmem_ld32(to + c * 32, v);
        if (tok < it.n) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 u = make_uint4(pack_bf16x2(v[q * 8 + 0] * inv, v[q * 8 + 1] * inv),
                                 pack_bf16x2(v[q * 8 + 2] * inv, v[q * 8 + 3] * inv),
                                 pack_bf16x2(v[q * 8 + 4] * inv, v[q * 8 + 5] * inv),
                                 pack_bf16x2(v[q * 8 + 6] * inv, v[q * 8 + 7] * inv));
            *reinterpret_cast<uint4*>(orow + c * 32 + q * 8) = u;
          }
        }
      }
      tc_fence_before();
      group_arrive(&bs->o_empty[w]);
    }
  }
  // teardown: the softmax warps waited for the last PV of their last item, and
  // that completion covers every earlier MMA of this CTA
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

// [heads][rows][D] bf16 (rows and heads at the given element strides) as a 3-D
// tensor map with a {64, box_rows, 1} box, 128-byte swizzle.
bool make_map(CUtensorMap* map, const void* base, int64_t rows, int32_t heads, int D, int box_rows, HeadTok st) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows),
                              static_cast<cuuint64_t>(heads)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(st.tok) * 2, static_cast<cuuint64_t>(st.head) * 2};
  const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int BLK>
cudaError_t launch_tc(const sws_handle* h, const void* q, const void* k, const void* v, int64_t n, int32_t hq,
                      int32_t hkv, const PrefillLayout& lay, const int32_t* row_ptr, const int32_t* col_idx, void* o,
                      cudaStream_t st) {
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, q, n, hq, D, kTileM, lay.q) || !make_map(&mk, k, n, hkv, D, BLK == 128 ? 128 : 64, lay.k) ||
      !make_map(&mv, v, n, hkv, D, BLK == 128 ? 128 : 64, lay.v))
    return cudaErrorInvalidValue;
  const size_t smem = Smem<D>::total + 1024;
  auto kern = attn_tc_kernel<D, BLK, false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int64_t b = ceil_div64(n, BLK);
  int64_t nnz = 0;
  for (int64_t i = 0; i < b; ++i) nnz += tau_of_row(i, h->cfg.density_num, h->cfg.density_den);
  const int64_t items = ceil_div64(n, 2 * kTileM) * hq;
  const int grid = static_cast<int>(std::min<int64_t>(items, h->num_sms));
  const float qscale = static_cast<float>(1.4426950408889634 / sqrt(static_cast<double>(D)));
  {
    const cudaError_t le =
        launch_k(kern, grid, kTcThreads, smem, st, mq, mk, mv, n, hq, hq / hkv, row_ptr, col_idx, nnz,
                 static_cast<__nv_bfloat16*>(o), lay.o, qscale, static_cast<const SeqDesc*>(nullptr),
                 static_cast<const int2*>(nullptr), 0, h->err);
    if (le != cudaSuccess) return le;
  }
  note_launches(1);
  return cudaGetLastError();
}

// Workspace of a packed launch: the sequence table, then the (sequence, slab)
// entries, longest slab first.
size_t varlen_table_bytes(int32_t nseq, const int64_t* cu) {
  int64_t ent = 0;
  for (int32_t s = 0; s < nseq; ++s) ent += ceil_div64(cu[s + 1] - cu[s], 2 * kTileM);
  return ((nseq * sizeof(SeqDesc) + 15) & ~size_t(15)) + static_cast<size_t>(ent) * sizeof(int2);
}

template <int D, int BLK>
cudaError_t launch_tc_var(const sws_handle* h, const void* q, const void* k, const void* v, int32_t hq, int32_t hkv,
                          const PrefillLayout& lay, int32_t nseq, const int64_t* cu, const int32_t* const* row_ptr,
                          const int32_t* const* col_idx, void* o, void* ws, cudaStream_t st) {
  const int64_t ntot = cu[nseq];
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, q, ntot, hq, D, kTileM, lay.q) || !make_map(&mk, k, ntot, hkv, D, BLK == 128 ? 128 : 64, lay.k) ||
      !make_map(&mv, v, ntot, hkv, D, BLK == 128 ? 128 : 64, lay.v))
    return cudaErrorInvalidValue;
  // the tables, built here and copied into the workspace in stream order (a
  // pageable source is staged before the call returns; no device wait)
  const size_t tab = (nseq * sizeof(SeqDesc) + 15) & ~size_t(15);
  std::vector<uint8_t> host(varlen_table_bytes(nseq, cu));
  SeqDesc* sd = reinterpret_cast<SeqDesc*>(host.data());
  int2* ent = reinterpret_cast<int2*>(host.data() + tab);
  int32_t max_slab = 0;
  for (int32_t s = 0; s < nseq; ++s) {
    const int64_t n = cu[s + 1] - cu[s], b = ceil_div64(n, BLK);
    int64_t nnz = 0;
    for (int64_t i = 0; i < b; ++i) nnz += tau_of_row(i, h->cfg.density_num, h->cfg.density_den);
    sd[s] = SeqDesc{row_ptr[s], col_idx[s], nnz, n, cu[s], b};
    max_slab = std::max(max_slab, static_cast<int32_t>(ceil_div64(n, 2 * kTileM)));
  }
  int32_t nent = 0;
  for (int32_t p = max_slab - 1; p >= 0; --p)  // longest slabs first, sequences in order within a length
    for (int32_t s = 0; s < nseq; ++s)
      if (ceil_div64(cu[s + 1] - cu[s], 2 * kTileM) > p) ent[nent++] = make_int2(s, p);
  cudaError_t e = cudaMemcpyAsync(ws, host.data(), host.size(), cudaMemcpyHostToDevice, st);
  if (e != cudaSuccess) return e;
  const size_t smem = Smem<D>::total + 1024;
  auto kern = attn_tc_kernel<D, BLK, true>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int64_t items = static_cast<int64_t>(nent) * hq;
  const int grid = static_cast<int>(std::min<int64_t>(items, h->num_sms));
  const float qscale = static_cast<float>(1.4426950408889634 / sqrt(static_cast<double>(D)));
  const auto* wsb = static_cast<const uint8_t*>(ws);
  {
    const cudaError_t le =
        launch_k(kern, grid, kTcThreads, smem, st, mq, mk, mv, ntot, hq, hq / hkv, static_cast<const int32_t*>(nullptr),
                 static_cast<const int32_t*>(nullptr), int64_t(0), static_cast<__nv_bfloat16*>(o), lay.o, qscale,
                 reinterpret_cast<const SeqDesc*>(wsb), reinterpret_cast<const int2*>(wsb + tab), nent, h->err);
    if (le != cudaSuccess) return le;
  }
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace

size_t attn_prefill_varlen_ws_bytes(int32_t nseq, const int64_t* cu_seqlens) {
  return varlen_table_bytes(nseq, cu_seqlens);
}

cudaError_t launch_attn_prefill_tc_varlen(const sws_handle* h, const void* q, const void* k, const void* v,
                                          int32_t hq, int32_t hkv, const PrefillLayout& lay, int32_t nseq,
                                          const int64_t* cu_seqlens, const int32_t* const* row_ptr,
                                          const int32_t* const* col_idx, void* o, void* ws, cudaStream_t st) {
  const int d = h->cfg.head_dim, B = h->cfg.block_size;
  if (d == 128) {
    return B == 128 ? launch_tc_var<128, 128>(h, q, k, v, hq, hkv, lay, nseq, cu_seqlens, row_ptr, col_idx, o, ws, st)
                    : launch_tc_var<128, 64>(h, q, k, v, hq, hkv, lay, nseq, cu_seqlens, row_ptr, col_idx, o, ws, st);
  }
  return B == 128 ? launch_tc_var<64, 128>(h, q, k, v, hq, hkv, lay, nseq, cu_seqlens, row_ptr, col_idx, o, ws, st)
                  : launch_tc_var<64, 64>(h, q, k, v, hq, hkv, lay, nseq, cu_seqlens, row_ptr, col_idx, o, ws, st);
}

cudaError_t launch_attn_prefill_tc(const sws_handle* h, const void* q, const void* k, const void* v, int64_t n,
                                   int32_t hq, int32_t hkv, const PrefillLayout& lay, const int32_t* row_ptr,
                                   const int32_t* col_idx, void* o, cudaStream_t st) {
  const int d = h->cfg.head_dim, B = h->cfg.block_size;
  if (d == 128) {
    return B == 128 ? launch_tc<128, 128>(h, q, k, v, n, hq, hkv, lay, row_ptr, col_idx, o, st)
                    : launch_tc<128, 64>(h, q, k, v, n, hq, hkv, lay, row_ptr, col_idx, o, st);
  }
  return B == 128 ? launch_tc<64, 128>(h, q, k, v, n, hq, hkv, lay, row_ptr, col_idx, o, st)
                  : launch_tc<64, 64>(h, q, k, v, n, hq, hkv, lay, row_ptr, col_idx, o, st);
}

}  // namespace sws
