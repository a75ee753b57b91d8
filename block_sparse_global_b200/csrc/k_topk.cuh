// Warp-level exact top-k selection shared by the selection kernels of libress.so: the c
// largest keys of a row, ties to the lower index, marked through a callback.
#pragma once

#include "ress_common.cuh"

namespace ress {

RESS_DEV int warp_sum_i(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
RESS_DEV unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Marks the k valid entries with the largest key (ties: lower index) by calling
// mark(j).  Warp-collective.  MSB-first radix select with 8-bit digits over a 256-bin
// shared-memory histogram (hist, this warp's); as soon as the bucket that holds the k-th
// key has at most 32 members, those members are gathered (slot: 32 ints of this warp's
// shared memory) and ranked exactly by (key descending, index ascending).
template <typename KeyT, typename KeyFn, typename ValidFn, typename MarkFn>
RESS_DEV void warp_top_k(int n, int k, KeyFn key, ValidFn valid, MarkFn mark, uint32_t *hist,
                         int *slot) {
  const int lane = threadIdx.x & 31;
  int nvalid = 0;
  for (int j = lane; j < n; j += 32) nvalid += valid(j) ? 1 : 0;
  nvalid = warp_sum_i(nvalid);
  if (k <= 0) return;
  if (k >= nvalid) {
    for (int j = lane; j < n; j += 32)
      if (valid(j)) mark(j);
    __syncwarp();
    return;
  }
  constexpr int BITS = sizeof(KeyT) * 8;
  KeyT prefix = 0;
  uint32_t remaining = (uint32_t)k, bucket = 0;
  int shift = BITS;
#pragma unroll 1
  while (shift > 0) {
    const int hi_shift = shift;  // bits above the digit being resolved
    shift -= 8;
    for (int b = lane; b < 256; b += 32) hist[b] = 0;
    __syncwarp();
    for (int base = 0; base < n; base += 32) {
      const int j = base + lane;
      bool in = j < n && valid(j);
      uint32_t bin = 0;
      if (in) {
        const KeyT kk = key(j);
        in = hi_shift >= BITS || (kk >> hi_shift) == (prefix >> hi_shift);
        bin = (uint32_t)(kk >> shift) & 255u;
      }
      // shared-memory atomics resolve lanes that hit the same bin in hardware
      if (in) atomicAdd(&hist[bin], 1u);
    }
    __syncwarp();
    // lane l holds bins 255-8l .. 248-8l (highest digits first)
    uint32_t cnt[8], tot = 0;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      cnt[q] = hist[255 - (lane * 8 + q)];
      tot += cnt[q];
    }
    uint32_t incl = tot;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    const uint32_t excl = incl - tot;
    const unsigned here = __ballot_sync(0xffffffffu, excl < remaining && remaining <= incl);
    const int src = __ffs(here) - 1;
    int digit = 0;
    uint32_t above = 0, inbin = 0;
    if (lane == src) {
      uint32_t acc = excl;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (acc + cnt[q] >= remaining) {
          digit = 255 - (lane * 8 + q);
          above = acc;
          inbin = cnt[q];
          break;
        }
        acc += cnt[q];
      }
    }
    digit = __shfl_sync(0xffffffffu, digit, src);
    above = __shfl_sync(0xffffffffu, above, src);
    bucket = __shfl_sync(0xffffffffu, inbin, src);
    remaining -= above;
    prefix |= KeyT(digit) << shift;
    __syncwarp();
    if (bucket <= 32) break;
  }
  // Keys whose bits at and above `shift` exceed the bucket's are taken; the bucket's
  // members are taken by rank.
  const KeyT top = prefix >> shift;
  uint32_t taken = 0;
  for (int base = 0; base < n; base += 32) {
    const int j = base + lane;
    const bool v = j < n && valid(j);
    const KeyT kt = v ? (key(j) >> shift) : KeyT(0);
    if (v && kt > top) mark(j);
    const bool inb = v && kt == top;
    const unsigned b = __ballot_sync(0xffffffffu, inb);
    if (bucket <= 32) {
      if (inb) slot[taken + __popc(b & lanemask_lt())] = j;
    } else if (inb && taken + __popc(b & lanemask_lt()) < remaining) {
      mark(j);  // all bits resolved: the bucket holds equal keys, take the lowest indices
    }
    taken += __popc(b);
  }
  __syncwarp();
  if (bucket <= 32) {
    const bool live = lane < (int)taken;
    const int j = live ? slot[lane] : 0;
    const KeyT kk = live ? key(j) : KeyT(0);
    uint32_t rank = 0;
    for (int m = 0; m < (int)taken; ++m) {
      const int jm = __shfl_sync(0xffffffffu, j, m);
      const KeyT km = __shfl_sync(0xffffffffu, kk, m);
      rank += (km > kk || (km == kk && jm < j)) ? 1u : 0u;
    }
    if (live && rank < remaining) mark(j);
  }
  __syncwarp();
}

// Marks the k entries q < n (n <= 64) with the largest key, ties to the lower q, by a
// direct rank: lane l holds entries l and l + 32 and counts, over all n entries, those
// that come before each of its own in (key descending, q ascending) order.  Same result
// as warp_top_k16 over the same entries, without histogram passes.
template <typename KeyFn, typename MarkFn>
RESS_DEV void warp_top_k_small(int n, int k, KeyFn key, MarkFn mark) {
  const int lane = threadIdx.x & 31;
  if (k <= 0 || n <= 0) return;
  const bool v0 = lane < n, v1 = lane + 32 < n;
  const uint32_t k0 = v0 ? key(lane) : 0u, k1 = v1 ? key(lane + 32) : 0u;
  uint32_t r0 = 0, r1 = 0;
  const int top = min(n, 32);
  for (int l = 0; l < top; ++l) {
    const uint32_t a = __shfl_sync(0xffffffffu, k0, l);  // entry l
    const uint32_t b = __shfl_sync(0xffffffffu, k1, l);  // entry l + 32
    const bool bv = l + 32 < n;
    r0 += (a > k0 || (a == k0 && l < lane)) ? 1u : 0u;
    r0 += (bv && b > k0) ? 1u : 0u;  // entry l + 32 comes after entry lane on a tie
    r1 += (a >= k1) ? 1u : 0u;       // entry l comes before entry lane + 32 on a tie
    r1 += (bv && (b > k1 || (b == k1 && l < lane))) ? 1u : 0u;
  }
  if (v0 && r0 < (uint32_t)k) mark(lane);
  if (v1 && r1 < (uint32_t)k) mark(lane + 32);
  __syncwarp();
}

// ---------------------------------------------------------------- 16-bit histograms
// A 256-bin histogram of 16-bit counts packed in 128 words (bin b in half b & 1 of word
// b >> 1); counts stay below 2^16 because a row has at most 4096 entries.
RESS_DEV void hist16_add(uint32_t *hist, uint32_t bin) {
  atomicAdd(&hist[bin >> 1], 1u << ((bin & 1u) * 16u));
}
RESS_DEV void hist16_clear(uint32_t *hist) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int w = lane; w < 128; w += 32) hist[w] = 0u;
}

// warp_top_k for 32-bit keys with the 16-bit histogram, for callers that know how many
// entries are valid (nvalid) and may have built the first pass's histogram already
// (first_done: hist holds the counts of every valid key's top byte).  Same result as
// warp_top_k: the k valid entries with the largest key, ties to the lower index.
template <typename KeyFn, typename ValidFn, typename MarkFn>
RESS_DEV void warp_top_k16(int n, int k, int nvalid, KeyFn key, ValidFn valid, MarkFn mark,
                           uint32_t *hist, int *slot, bool first_done) {
  const int lane = threadIdx.x & 31;
  if (k <= 0) return;
  if (k >= nvalid) {
    for (int j = lane; j < n; j += 32)
      if (valid(j)) mark(j);
    __syncwarp();
    return;
  }
  uint32_t prefix = 0, remaining = (uint32_t)k, bucket = 0;
  int shift = 32;
  bool have = first_done;
#pragma unroll 1
  while (shift > 0) {
    const int hi_shift = shift;
    shift -= 8;
    if (!have) {
      hist16_clear(hist);
      __syncwarp();
      for (int base = 0; base < n; base += 32) {
        const int j = base + lane;
        if (j < n && valid(j)) {
          const uint32_t kk = key(j);
          if (hi_shift >= 32 || (kk >> hi_shift) == (prefix >> hi_shift)) hist16_add(hist, (kk >> shift) & 255u);
        }
      }
      __syncwarp();
    }
    have = false;
    // lane l holds bins 255-8l .. 248-8l (highest digits first)
    uint32_t cnt[8], tot = 0;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const uint32_t b = 255u - (uint32_t)(lane * 8 + q);
      cnt[q] = (hist[b >> 1] >> ((b & 1u) * 16u)) & 0xFFFFu;
      tot += cnt[q];
    }
    uint32_t incl = tot;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    const uint32_t excl = incl - tot;
    const unsigned here = __ballot_sync(0xffffffffu, excl < remaining && remaining <= incl);
    const int src = __ffs(here) - 1;
    int digit = 0;
    uint32_t above = 0, inbin = 0;
    if (lane == src) {
      uint32_t acc = excl;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (acc + cnt[q] >= remaining) {
          digit = 255 - (lane * 8 + q);
          above = acc;
          inbin = cnt[q];
          break;
        }
        acc += cnt[q];
      }
    }
    digit = __shfl_sync(0xffffffffu, digit, src);
    above = __shfl_sync(0xffffffffu, above, src);
    bucket = __shfl_sync(0xffffffffu, inbin, src);
    remaining -= above;
    prefix |= (uint32_t)digit << shift;
    __syncwarp();
    if (bucket <= 32) break;
  }
  const uint32_t top = prefix >> shift;
  uint32_t taken = 0;
  for (int base = 0; base < n; base += 32) {
    const int j = base + lane;
    const bool v = j < n && valid(j);
    const uint32_t kt = v ? (key(j) >> shift) : 0u;
    if (v && kt > top) mark(j);
    const bool inb = v && kt == top;
    const unsigned b = __ballot_sync(0xffffffffu, inb);
    if (bucket <= 32) {
      if (inb) slot[taken + __popc(b & lanemask_lt())] = j;
    } else if (inb && taken + __popc(b & lanemask_lt()) < remaining) {
      mark(j);
    }
    taken += __popc(b);
  }
  __syncwarp();
  if (bucket <= 32) {
    const bool live = lane < (int)taken;
    const int j = live ? slot[lane] : 0;
    const uint32_t kk = live ? key(j) : 0u;
    uint32_t rank = 0;
    for (int m = 0; m < (int)taken; ++m) {
      const int jm = __shfl_sync(0xffffffffu, j, m);
      const uint32_t km = __shfl_sync(0xffffffffu, kk, m);
      rank += (km > kk || (km == kk && jm < j)) ? 1u : 0u;
    }
    if (live && rank < remaining) mark(j);
  }
  __syncwarp();
}

// Marks the k valid entries with the largest key (ties: lower index) for small k by
// repeated warp-wide arg-max: every lane keeps the best of its own entries (j = lane,
// lane + 32, ...), the warp picks the best of the 32, its owner marks it (which makes it
// invalid) and rescans its own entries.  Exact, and cheap while k is small.
template <typename KeyT, typename KeyFn, typename ValidFn, typename MarkFn>
RESS_DEV void warp_top_k_extract(int n, int k, KeyFn key, ValidFn valid, MarkFn mark) {
  const int lane = threadIdx.x & 31;
  auto local_best = [&](KeyT &bk, int &bj) {
    bj = -1;
    bk = KeyT(0);
    for (int j = lane; j < n; j += 32) {
      if (!valid(j)) continue;
      const KeyT kk = key(j);
      if (bj < 0 || kk > bk) {  // ascending scan: a tie keeps the lower index
        bk = kk;
        bj = j;
      }
    }
  };
  KeyT bk;
  int bj;
  local_best(bk, bj);
  for (int r = 0; r < k; ++r) {
    KeyT wk = bk;
    int wj = bj;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const KeyT ok = __shfl_xor_sync(0xffffffffu, wk, o);
      const int oj = __shfl_xor_sync(0xffffffffu, wj, o);
      const bool better = oj >= 0 && (wj < 0 || ok > wk || (ok == wk && oj < wj));
      if (better) {
        wk = ok;
        wj = oj;
      }
    }
    if (wj < 0) break;  // fewer valid entries than k
    if (lane == (wj & 31)) {
      mark(wj);
      local_best(bk, bj);
    }
    __syncwarp();
  }
  __syncwarp();
}

// Exact top-k: extraction while k is small, radix select otherwise.
template <typename KeyT, typename KeyFn, typename ValidFn, typename MarkFn>
RESS_DEV void warp_select(int n, int k, KeyFn key, ValidFn valid, MarkFn mark, uint32_t *hist,
                          int *slot) {
  if (k <= 4)
    warp_top_k_extract<KeyT>(n, k, key, valid, mark);
  else
    warp_top_k<KeyT>(n, k, key, valid, mark, hist, slot);
}

// Eq. 17 swap count: max(1, round-half-up(rho c 2^-(r+1))), capped at |D| and c.

// CDF / top-p cut after a top-c by probability (SparseVGGT's rule): of the kept entries,
// in (pv descending, index ascending) order, keep the shortest prefix whose sum plus
// fixed_mass reaches top_p (float64 partial sums), at least one.  pv[j] is entry j's
// probability, kept(j) / unkeep(j) read and clear its kept state, sorted is warp scratch
// for at least as many floats as entries are kept.  Warp-collective.
template <typename KeptFn, typename UnkeepFn>
RESS_DEV void warp_cdf_cut(int n, const float *pv, KeptFn kept, UnkeepFn unkeep, double fixed_mass,
                           float top_p, float *sorted) {
  const int lane = threadIdx.x & 31;
  auto rank_of = [&](int j) {
    const float x = pv[j];
    int r = 0;
    for (int k = 0; k < n; ++k)
      if (kept(k)) {
        const float y = pv[k];
        r += (y > x || (y == x && k < j)) ? 1 : 0;
      }
    return r;
  };
  int c = 0;
  for (int j = lane; j < n; j += 32)
    if (kept(j)) {
      sorted[rank_of(j)] = pv[j];
      ++c;
    }
  c = warp_sum_i(c);
  __syncwarp();
  // first position whose running sum (plus the always-kept mass) reaches top_p
  int cut = c;
  double run = fixed_mass;
  for (int base = 0; base < c; base += 32) {
    const int q = base + lane;
    double incl = q < c ? (double)sorted[q] : 0.0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const double y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const unsigned hit = __ballot_sync(0xffffffffu, q < c && run + incl >= (double)top_p);
    if (hit) {
      cut = base + __ffs(hit);
      break;
    }
    run += __shfl_sync(0xffffffffu, incl, 31);
  }
  cut = max(1, cut);
  // decide every drop against the unchanged kept set, then apply (n <= 4096: at most
  // 128 entries per lane).  Entries above the value at the cut stay, entries below it
  // go; only entries equal to it need their rank.
  const float vcut = sorted[cut - 1];
  uint32_t drop[4] = {0u, 0u, 0u, 0u};
  for (int j = lane, t = 0; j < n; j += 32, ++t)
    if (kept(j)) {
      const float x = pv[j];
      if (x < vcut || (x == vcut && rank_of(j) >= cut)) drop[t >> 5] |= 1u << (t & 31);
    }
  __syncwarp();
  for (int j = lane, t = 0; j < n; j += 32, ++t)
    if (drop[t >> 5] & (1u << (t & 31))) unkeep(j);
  __syncwarp();
}

}  // namespace ress
