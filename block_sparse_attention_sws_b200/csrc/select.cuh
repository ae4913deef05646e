// Warp-level exact top-tau selection (radix select on 64-bit keys).
//
// "Scout Before You Attend" §4: for each query block, the tau key blocks with the
// largest walk score. Ties go to the lower block index and the chosen indices are
// written in ascending order.
#pragma once

#include "sws_common.cuh"

namespace sws {

// Order-preserving map from a double to an unsigned 64-bit key.
__device__ __forceinline__ uint64_t order_key(double x) {
  const uint64_t u = static_cast<uint64_t>(__double_as_longlong(x));
  return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}

__device__ __forceinline__ unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// keys[0, m): shared memory, written before the call and visible to the warp.
// Writes the tau chosen indices, ascending, to out[0, tau) (1 <= tau <= m).
// An 8-bit radix select: up to eight passes, each counting the keys that still
// match the prefix found so far in a 256-bin histogram hist[] (shared memory
// owned by this warp); then an ordered compaction in index order that takes
// every key above the threshold and the first `need` keys equal to it.
__device__ __forceinline__ void warp_top_tau8(const uint64_t* keys, int m, int tau, int32_t* out, int* hist,
                                              int32_t* err) {
  const int lane = threadIdx.x & 31;
  uint64_t prefix = 0, pmask = 0;
  int need = tau;
  bool all_cands = false;
  for (int shift = 56; shift >= 0; shift -= 8) {
#pragma unroll
    for (int u = 0; u < 8; ++u) hist[lane * 8 + u] = 0;
    __syncwarp();
    for (int j = lane; j < m; j += 32) {
      const uint64_t key = keys[j];
      if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1);
    }
    __syncwarp();
    // lane l owns bins 255 - 8 l - u (u = 0..7), in descending key order
    int c[8], sum = 0;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      c[u] = hist[255 - 8 * lane - u];
      sum += c[u];
    }
    int incl = sum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += y;
    }
    const int excl = incl - sum;
    int digit = 0, rest = 0, cnt = 0;
    const bool here = excl < need && need <= incl;
    if (here) {
      int run = excl;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        if (run + c[u] >= need) {
          digit = 255 - 8 * lane - u;
          rest = need - run;
          cnt = c[u];
          break;
        }
        run += c[u];
      }
    }
    const unsigned who = __ballot_sync(0xffffffffu, here);
    const int src = who ? __ffs(who) - 1 : 0;
    digit = __shfl_sync(0xffffffffu, digit, src);
    rest = __shfl_sync(0xffffffffu, rest, src);
    cnt = __shfl_sync(0xffffffffu, cnt, src);
    __syncwarp();  // every lane has read hist before the next pass clears it
    prefix |= static_cast<uint64_t>(digit) << shift;
    pmask |= 255ull << shift;
    need = rest;
    if (cnt == need) {
      all_cands = true;
      break;
    }
  }
  const unsigned lt = lanemask_lt();
  int base = 0, ties = 0;
  for (int j0 = 0; j0 < m; j0 += 32) {
    const int j = j0 + lane;
    const bool valid = j < m;
    const uint64_t km = valid ? (keys[j] & pmask) : 0;
    const bool above = valid && km > prefix;
    const bool cand = valid && km == prefix;
    const unsigned cb = __ballot_sync(0xffffffffu, cand);
    bool take = cand;
    if (!all_cands) {
      take = cand && (ties + __popc(cb & lt)) < need;
      ties += __popc(cb);
    }
    const bool sel = above || take;
    const unsigned sb = __ballot_sync(0xffffffffu, sel);
    if (sel) {
      const int pos = base + __popc(sb & lt);
      if (pos < tau) out[pos] = j;
    }
    base += __popc(sb);
  }
  if (lane == 0 && base != tau) record_error(err, GUARD_BAD_SELECT);
}

// ---- helpers shared by the decode-side kernels ------------------------------

__device__ __forceinline__ void named_bar(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Output o of a length-D row times H_d, computed by one warp: lane l sums the
// terms t = l, l + 32, ..., then a shuffle tree adds the lanes.
template <int D>
__device__ __forceinline__ double warp_dot_hdt(const double* row_smem, const double* __restrict__ hdt_row, int lane) {
  double a = 0.0;
#pragma unroll
  for (int t = lane; t < D; t += 32) a = fma(row_smem[t], __ldg(hdt_row + t), a);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) a += __shfl_xor_sync(0xffffffffu, a, off);
  return a;
}

// Exact top-tau of keys[0, m) (ties to the lower index) by nthr threads (whole
// warps, the first of them warp `w0`) that share named barrier `bar_id`:
// eight passes of an 8-bit radix select on the 64-bit keys (a 256-bin shared
// histogram of the keys that still match the prefix found so far), then an
// ordered compaction by the first warp that writes the chosen indices
// ascending to out[] and ORs `bit` into mark[j].
__device__ inline void group_top_tau(const uint64_t* keys, int m, int tau, int* hist, int* ctl, int t, int nthr,
                                     int bar_id, int32_t* out, uint32_t* mark, uint32_t bit, int32_t* err) {
  uint64_t prefix = 0, pm = 0;
  int need = tau;
  bool all_cands = false;
  for (int shift = 56; shift >= 0; shift -= 8) {
    for (int x = t; x < 256; x += nthr) hist[x] = 0;
    if (t == 0) ctl[0] = ctl[1] = ctl[2] = 0;
    named_bar(bar_id, nthr);
    for (int j = t; j < m; j += nthr) {
      const uint64_t key = keys[j];
      if ((key & pm) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1);
    }
    named_bar(bar_id, nthr);
    if (t < 32) {
      // lane l owns bins 255 - 8l - u, u = 0..7 (descending key order)
      int c[8], sum = 0;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        c[u] = hist[255 - 8 * t - u];
        sum += c[u];
      }
      int incl = sum;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, off);
        if (t >= off) incl += y;
      }
      const int excl = incl - sum;
      if (excl < need && need <= incl) {
        int run = excl;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          if (run + c[u] >= need) {
            ctl[0] = 255 - 8 * t - u;
            ctl[1] = need - run;
            ctl[2] = c[u];
            break;
          }
          run += c[u];
        }
      }
    }
    named_bar(bar_id, nthr);
    const int digit = ctl[0];
    need = ctl[1];
    const int cnt = ctl[2];
    prefix |= static_cast<uint64_t>(digit) << shift;
    pm |= 255ull << shift;
    named_bar(bar_id, nthr);  // ctl and hist are rewritten by the next pass
    if (cnt == need) {
      all_cands = true;
      break;
    }
  }
  if (t >= 32) return;
  const unsigned lt = lanemask_lt();
  int base = 0, ties = 0;
  for (int j0 = 0; j0 < m; j0 += 32) {
    const int j = j0 + t;
    const bool valid = j < m;
    const uint64_t km = valid ? (keys[j] & pm) : 0;
    const bool above = valid && km > prefix;
    const bool cand = valid && km == prefix;
    const unsigned cb = __ballot_sync(0xffffffffu, cand);
    bool take = cand;
    if (!all_cands) {
      take = cand && (ties + __popc(cb & lt)) < need;
      ties += __popc(cb);
    }
    const bool sel = above || take;
    const unsigned sb = __ballot_sync(0xffffffffu, sel);
    if (sel) {
      const int pos = base + __popc(sb & lt);
      if (pos < tau) out[pos] = j;
      atomicOr(&mark[j], bit);
    }
    base += __popc(sb);
  }
  if (t == 0 && base != tau) record_error(err, GUARD_BAD_SELECT);
}

}  // namespace sws
