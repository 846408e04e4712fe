// topk_select.cuh -- block-wide radix select used by the top-k selector
// ("DeepSeek-V4 内部机制" 1.2 Step 2 and 6.2: top-k over the BF16 index score).
//
// Keys are order-preserving 32-bit images of the scores (bf16 scores occupy
// the upper 16 bits, so they need two 8-bit digit passes; fp32 scores need
// four).  The selection order is (key desc, position asc): after the digit
// passes fix the k-th key T, every key > T is taken and the first keys == T in
// position order fill the remaining slots, which breaks ties toward the lower
// entry index because positions follow entry indices.
#pragma once

#include <stdint.h>

namespace csa {

template <int NT>
struct SelectSmem {
  uint32_t hist[256];
  uint32_t warp_tot[NT / 32];
  uint32_t bcast[4];
};

// Exclusive block-wide prefix sum of one value per thread; returns the total
// through `total`.  All NT threads must call it.
template <int NT>
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, uint32_t* warp_tot,
                                                         uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tot[warp] = x;
  __syncthreads();
  if (warp == 0) {
    uint32_t t = lane < NT / 32 ? warp_tot[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      uint32_t y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    if (lane < NT / 32) warp_tot[lane] = t;  // inclusive
  }
  __syncthreads();
  const uint32_t before = (warp > 0 ? warp_tot[warp - 1] : 0) + x - v;
  *total = warp_tot[NT / 32 - 1];
  __syncthreads();
  return before;
}

// Radix threshold: finds the key T of the kk-th largest key among positions
// [0, n) and the number `need_eq` of keys equal to T that belong to the top kk.
// `key_at(i)` returns the key at position i.  passes = 2 (bf16 keys) or 4.
template <int NT, class KeyAt>
__device__ void radix_threshold(const KeyAt& key_at, int n, int kk, int passes,
                                SelectSmem<NT>& sm, uint32_t* T_out, int* need_eq_out) {
  uint32_t prefix = 0, mask = 0;
  int remaining = kk;
  for (int p = 0; p < passes; ++p) {
    const int shift = 24 - 8 * p;
    for (int i = threadIdx.x; i < 256; i += NT) sm.hist[i] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += NT) {
      const uint32_t key = key_at(i);
      if ((key & mask) == prefix) atomicAdd(&sm.hist[(key >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      const int lane = threadIdx.x;
      // lane l covers digits 255-8l .. 248-8l (descending)
      uint32_t c[8], s = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) { c[j] = sm.hist[255 - 8 * lane - j]; s += c[j]; }
      uint32_t inc = s;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += y;
      }
      const uint32_t exc = inc - s;
      const bool here = exc < (uint32_t)remaining && (uint32_t)remaining <= inc;
      const unsigned ballot = __ballot_sync(0xffffffffu, here);
      if (here && lane == __ffs(ballot) - 1) {
        uint32_t above = exc;
        int digit = 255 - 8 * lane;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (above + c[j] >= (uint32_t)remaining) { digit = 255 - 8 * lane - j; break; }
          above += c[j];
        }
        sm.bcast[0] = (uint32_t)digit;
        sm.bcast[1] = (uint32_t)remaining - above;
      }
    }
    __syncthreads();
    prefix |= sm.bcast[0] << shift;
    mask |= 255u << shift;
    remaining = (int)sm.bcast[1];
    __syncthreads();
  }
  *T_out = prefix;
  *need_eq_out = remaining;
}

// Writes the top kk (key desc, position asc) of positions [0, n) in ascending
// position order through emit(out_slot, position).  Requires kk <= n.
template <int NT, class KeyAt, class Emit>
__device__ void block_select(const KeyAt& key_at, int n, int kk, int passes, SelectSmem<NT>& sm,
                             const Emit& emit) {
  if (kk <= 0) return;
  if (kk >= n) {  // everything is selected
    for (int i = threadIdx.x; i < n; i += NT) emit(i, i);
    return;
  }
  uint32_t T;
  int need_eq;
  radix_threshold<NT>(key_at, n, kk, passes, sm, &T, &need_eq);
  const int chunk = (n + NT - 1) / NT;
  const int i0 = min(n, (int)threadIdx.x * chunk), i1 = min(n, i0 + chunk);
  uint32_t c_gt = 0, c_eq = 0;
  for (int i = i0; i < i1; ++i) {
    const uint32_t key = key_at(i);
    c_gt += key > T;
    c_eq += key == T;
  }
  uint32_t tot;
  const uint32_t eq_before = block_exclusive_scan<NT>(c_eq, sm.warp_tot, &tot);
  int eq_take = need_eq - (int)eq_before;
  eq_take = eq_take < 0 ? 0 : (eq_take > (int)c_eq ? (int)c_eq : eq_take);
  const uint32_t out_before = block_exclusive_scan<NT>(c_gt + (uint32_t)eq_take, sm.warp_tot, &tot);
  uint32_t o = out_before;
  int eq_seen = 0;
  for (int i = i0; i < i1; ++i) {
    const uint32_t key = key_at(i);
    bool take = key > T;
    if (key == T) { take = eq_seen < eq_take; ++eq_seen; }
    if (take) emit((int)o++, i);
  }
}

}  // namespace csa
