// topk_select.cuh -- block-wide radix select used by the top-k selector
// ("DeepSeek-V4 内部机制" 1.2 Step 2 and 6.2: top-k over the BF16 index score).
//
// Keys are order-preserving 32-bit images of the scores (bf16 scores occupy
// the upper 16 bits).  The selection order is (key desc, position asc): after
// the digit passes fix the k-th key T, every key > T is taken and the first
// keys == T in position order fill the remaining slots, which breaks ties
// toward the lower entry index because positions follow entry indices.
//
// Range-adaptive digits: the keys of one row cluster in a narrow band (a few
// bf16 exponents), so fixed 8-bit digits would put almost every key into one
// or two histogram bins and serialise the shared-memory atomics.  The select
// first finds the band [lo, hi] of the candidate keys and works on the
// renormalised keys (key - lo) << (32 - bits), bits = bit length of hi - lo,
// whose leading 8-bit digits spread over the band.
#pragma once

#include <stdint.h>

namespace csa {

template <int NT>
struct SelectSmem {
  uint32_t hist[256];
  uint32_t warp_tot[NT / 32];
  uint32_t bcast[4];
};

// Radix threshold over renormalised keys: finds the kk-th largest rel key T
// among the valid positions and the number `need_eq` of keys equal to T that
// belong to the top kk.  rel(i, valid) returns the renormalised key at
// position i and whether the position takes part.
template <int NT, class Rel>
__device__ void radix_threshold(const Rel& rel, int n, int kk, int passes, SelectSmem<NT>& sm, uint32_t* T_out,
                                int* need_eq_out) {
  uint32_t prefix = 0, mask = 0;
  int remaining = kk;
  for (int p = 0; p < passes; ++p) {
    const int shift = 24 - 8 * p;
    for (int i = threadIdx.x; i < 256; i += NT) sm.hist[i] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += NT) {
      bool valid;
      const uint32_t key = rel(i, valid);
      if (valid && (key & mask) == prefix) atomicAdd(&sm.hist[(key >> shift) & 255u], 1u);
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
// position order through emit(out_slot, position).  Keys below `floor` never
// take part; the caller guarantees that at least kk keys are >= floor (kk <=
// n).  *T_out (optional) receives the kk-th largest key, or 0 when every
// position is selected.
//
// Compaction: warp w owns the contiguous positions [w*span, (w+1)*span) and
// walks them 32 at a time (coalesced); ballots rank the taken positions inside
// each step, and the per-warp counts order the warps, so the output follows
// position order and ties at T go to the lowest positions.
template <int NT, class KeyAt, class Emit>
__device__ void block_select(const KeyAt& key_at, int n, int kk, int /*unused*/, SelectSmem<NT>& sm,
                             const Emit& emit, uint32_t floor = 0, uint32_t* T_out = nullptr) {
  constexpr int NW = NT / 32;
  if (kk <= 0 || kk >= n) {  // nothing or everything is selected
    for (int i = threadIdx.x; i < n && kk > 0; i += NT) emit(i, i);
    if (T_out) *T_out = 0;
    return;
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  // band of the candidate keys
  uint32_t lo = 0xffffffffu, hi = 0u;
  for (int i = threadIdx.x; i < n; i += NT) {
    const uint32_t k = key_at(i);
    if (k >= floor) { lo = min(lo, k); hi = max(hi, k); }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  if (lane == 0) { sm.hist[warp] = lo; sm.hist[128 + warp] = hi; }
  __syncthreads();
  lo = 0xffffffffu;
  hi = 0u;
  for (int w = 0; w < NW; ++w) { lo = min(lo, sm.hist[w]); hi = max(hi, sm.hist[128 + w]); }
  __syncthreads();
  const int bits = hi > lo ? 32 - __clz(hi - lo) : 0;
  const int sh = 32 - bits;
  auto rel = [&](int i, bool& valid) -> uint32_t {
    const uint32_t k = key_at(i);
    valid = k >= floor;
    return (valid && bits > 0) ? (k - lo) << sh : 0u;
  };
  uint32_t Trel = 0;
  int need_eq = kk;
  if (bits > 0) radix_threshold<NT>(rel, n, kk, (bits + 7) / 8, sm, &Trel, &need_eq);
  if (T_out) *T_out = bits > 0 ? lo + (Trel >> sh) : lo;
  const unsigned lt = (1u << lane) - 1u;
  const int span = ((n + NW - 1) / NW + 31) / 32 * 32;
  const int w0 = min(n, warp * span), w1 = min(n, w0 + span);
  uint32_t c_gt = 0, c_eq = 0;
  for (int base = w0; base < w1; base += 32) {
    const int i = base + lane;
    bool valid = false;
    const uint32_t key = i < w1 ? rel(i, valid) : 0u;
    c_gt += __popc(__ballot_sync(0xffffffffu, valid && key > Trel));
    c_eq += __popc(__ballot_sync(0xffffffffu, valid && key == Trel));
  }
  // per-warp (gt, eq) counts -> ordered offsets
  if (lane == 0) sm.warp_tot[warp] = c_eq;
  __syncthreads();
  uint32_t eq_before = 0;
  for (int w = 0; w < warp; ++w) eq_before += sm.warp_tot[w];
  int eq_take = need_eq - (int)eq_before;
  eq_take = eq_take < 0 ? 0 : (eq_take > (int)c_eq ? (int)c_eq : eq_take);
  __syncthreads();
  if (lane == 0) sm.warp_tot[warp] = c_gt + (uint32_t)eq_take;
  __syncthreads();
  uint32_t o = 0;
  for (int w = 0; w < warp; ++w) o += sm.warp_tot[w];
  __syncthreads();
  int eq_seen = 0;
  for (int base = w0; base < w1; base += 32) {
    const int i = base + lane;
    bool valid = false;
    const uint32_t key = i < w1 ? rel(i, valid) : 0u;
    const unsigned eqm = __ballot_sync(0xffffffffu, valid && key == Trel);
    const bool take = valid && (key > Trel || (key == Trel && eq_seen + __popc(eqm & lt) < eq_take));
    const unsigned tm = __ballot_sync(0xffffffffu, take);
    if (take) emit((int)(o + __popc(tm & lt)), i);
    o += __popc(tm);
    eq_seen += __popc(eqm);
  }
}

}  // namespace csa
