// Device helpers shared by the HISA kernels (sm_100a).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#define HSA_DEV __device__ __forceinline__

namespace hsa {

constexpr unsigned kFull = 0xffffffffu;

// bf16 halves of a 32-bit word (little endian: element 0 in the low half).
HSA_DEV float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
HSA_DEV float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Round-to-nearest-even fp32 -> bf16 bits.
HSA_DEV uint32_t f32_to_bf16_rn(float f) {
  uint32_t u = __float_as_uint(f);
  u += 0x7fffu + ((u >> 16) & 1u);
  return u >> 16;
}
// Same rounding (nearest, ties to even) with the hardware convert.
HSA_DEV uint32_t cvt_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Order-preserving unsigned key of an fp32 score: larger score -> larger key.
// -0 is folded onto +0 so that the two compare equal, as floats do.
HSA_DEV uint32_t score_key(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u << 1) == 0u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
// Programmatic dependent launch. A kernel launched with the attribute may
// start while the previous kernel of its stream is still running; it calls
// griddep_wait() before touching any memory that kernel reads or writes (the
// wait returns once that kernel has completed and its writes are visible; it
// is a no-op for a normal launch), then griddep_launch() to let the next
// kernel of the stream start its own launch.
HSA_DEV void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
HSA_DEV void griddep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// The score a key stands for (inverse of score_key; -0 comes back as +0).
HSA_DEV float key_score(uint32_t u) { return __uint_as_float((u & 0x80000000u) ? (u & 0x7fffffffu) : ~u); }

// Which absolute position a query row has, and where its sequence lives.
// Prefill: one sequence, query row i is position Lk - Lq + i.
// Decode: row i is sequence i, at position ctx[i], with `capacity` cached
// rows per sequence.
struct RowMap {
  int64_t Lq, Lk;
  const int32_t* ctx;
  int64_t capacity;
  HSA_DEV int64_t pos(int64_t i) const { return ctx ? int64_t(ctx[i]) : Lk - Lq + i; }
  HSA_DEV int64_t seq_row0(int64_t i) const { return ctx ? i * capacity : 0; }
  HSA_DEV bool valid(int64_t i) const { return ctx ? (ctx[i] >= 0 && int64_t(ctx[i]) < capacity) : true; }
};

// Block-wide exclusive scan of one int per thread. Returns the exclusive
// prefix and writes the block total to *total. s_tmp holds >= NT/32 + 1 ints.
template <int NT>
HSA_DEV int block_exclusive_scan(int v, int* s_tmp, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(kFull, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) s_tmp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = lane < NT / 32 ? s_tmp[lane] : 0;
    int z = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(kFull, z, o);
      if (lane >= o) z += y;
    }
    if (lane < NT / 32) s_tmp[lane] = z - w;
    if (lane == NT / 32 - 1) s_tmp[NT / 32] = z;
  }
  __syncthreads();
  int res = s_tmp[warp] + x - v;
  *total = s_tmp[NT / 32];
  __syncthreads();
  return res;
}

// Block-wide exclusive scan in reverse thread order: thread t gets the sum
// of v over threads t+1 .. NT-1.
template <int NT>
HSA_DEV int block_exclusive_scan_rev(int v, int* s_tmp, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;  // inclusive suffix sum within the warp
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_down_sync(kFull, x, o);
    if (lane + o < 32) x += y;
  }
  if (lane == 0) s_tmp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = lane < NT / 32 ? s_tmp[lane] : 0;
    int z = w;  // inclusive suffix over warps
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_down_sync(kFull, z, o);
      if (lane + o < 32) z += y;
    }
    if (lane < NT / 32) s_tmp[lane] = z - w;
    if (lane == 0) s_tmp[NT / 32] = z;
  }
  __syncthreads();
  int res = s_tmp[warp] + x - v;
  *total = s_tmp[NT / 32];
  __syncthreads();
  return res;
}

// CTA-wide selection of the r largest of n keys (1 <= r <= n, keys in
// shared memory), ties broken towards the lowest position.
// threshold(): the r-th largest key T is found by histogramming the keys
// relative to their minimum in 2048 bins over the [min, max] range, then
// narrowing to the bin holding the r-th largest and repeating on that bin
// (11 bits per round, so at most three rounds; one round when the keys span
// fewer than 2048 values). take_eq = how many keys equal to T are taken.
// compact(): emits every selected position in ascending order: all keys > T
// and the first take_eq keys == T.
template <int NT>
struct RadixSelect {
  static constexpr int kBins = 2048;
  static_assert(kBins % NT == 0, "bins per thread");
  uint32_t* hist;   // smem, kBins entries
  int* scratch;     // smem, NT/32 + 8 ints

  HSA_DEV void threshold(const uint32_t* keys, int n, int r, uint32_t* T_out, int* take_eq) {
    constexpr int NW = NT / 32, BPT = kBins / NT;
    const int lane = threadIdx.x & 31;
    volatile int* s = scratch + NW + 2;  // [0]: min, [1]: max, [2]: bin, [3]: above
    uint32_t lo = 0xffffffffu, hi = 0u;
    for (int c = threadIdx.x; c < n; c += NT) { const uint32_t u = keys[c]; lo = min(lo, u); hi = max(hi, u); }
    lo = __reduce_min_sync(kFull, lo);
    hi = __reduce_max_sync(kFull, hi);
    if (threadIdx.x == 0) { s[0] = int(0xffffffffu); s[1] = 0; }
    __syncthreads();
    if (lane == 0) { atomicMin((unsigned*)&s[0], lo); atomicMax((unsigned*)&s[1], hi); }
    __syncthreads();
    uint32_t base = uint32_t(s[0]);
    uint32_t width = uint32_t(s[1]) - base;  // keys of interest lie in [base, base + width]
    int rem = r;
    for (;;) {
      const int bits = 32 - __clz(width);    // bits needed for (key - base)
      const int shift = bits > 11 ? bits - 11 : 0;
      for (int e = threadIdx.x; e < kBins; e += NT) hist[e] = 0;
      __syncthreads();
      const int per = ((n + NT - 1) / NT);
      for (int it = 0; it < per; ++it) {
        const int c = it * NT + threadIdx.x;
        const uint32_t u = c < n ? keys[c] : 0u;
        const bool in = c < n && u - base <= width;
        const uint32_t bin = in ? (u - base) >> shift : 0xffffffffu;
        const unsigned same = __match_any_sync(kFull, bin);
        if (in && lane == __ffs(same) - 1) atomicAdd(&hist[bin], __popc(same));
      }
      __syncthreads();
      // bins above each thread's BPT bins, via a scan over threads in reverse
      uint32_t cnt[BPT], tot = 0;
#pragma unroll
      for (int e = 0; e < BPT; ++e) { cnt[e] = hist[threadIdx.x * BPT + e]; tot += cnt[e]; }
      int total;
      // exclusive scan in reversed thread order = counts of all bins above mine
      int above = block_exclusive_scan_rev<NT>(int(tot), scratch, &total);
      if (uint32_t(above) < uint32_t(rem) && uint32_t(rem) <= uint32_t(above) + tot) {
        uint32_t a = uint32_t(above);
        for (int e = BPT - 1; e >= 0; --e) {
          if (a + cnt[e] >= uint32_t(rem)) { s[2] = threadIdx.x * BPT + e; s[3] = int(a); break; }
          a += cnt[e];
        }
      }
      __syncthreads();
      const uint32_t bin = uint32_t(s[2]);
      rem -= s[3];
      base += bin << shift;
      const uint32_t span = shift ? ((1u << shift) - 1u) : 0u;
      width = min(span, uint32_t(s[1]) - base);
      __syncthreads();
      if (shift == 0) break;
    }
    *T_out = base;
    *take_eq = rem;
  }

  // Emits (rank, pos) for every selected position, ascending. Warps own
  // contiguous position ranges; lanes interleave inside them. A position's
  // rank is (#keys > T before it) + min(#keys == T before it, take_eq).
  template <class Emit>
  HSA_DEV void compact(const uint32_t* keys, int n, uint32_t T, int take_eq, Emit emit) {
    constexpr int NW = NT / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int per = ((n + NW * 32 - 1) / (NW * 32)) * 32;
    const int lo = warp * per, hi = min(n, lo + per);
    int ngt = 0, neq = 0;
    for (int c0 = lo; c0 < hi; c0 += 32) {
      const int c = c0 + lane;
      const uint32_t u = c < hi ? keys[c] : 0u;
      ngt += __popc(__ballot_sync(kFull, c < hi && u > T));
      neq += __popc(__ballot_sync(kFull, c < hi && u == T));
    }
    int tot;
    // one scan over the packed pair (counts < 2^15 per CTA for n <= 16384)
    const int packed = block_exclusive_scan<NT>(lane == 0 ? (ngt << 16) | neq : 0, scratch, &tot);
    const int pk = __shfl_sync(kFull, packed, 0);
    int gt_before = pk >> 16, eq_before = pk & 0xffff;
    for (int c0 = lo; c0 < hi; c0 += 32) {
      const int c = c0 + lane;
      const uint32_t u = c < hi ? keys[c] : 0u;
      const unsigned bgt = __ballot_sync(kFull, c < hi && u > T);
      const unsigned beq = __ballot_sync(kFull, c < hi && u == T);
      const unsigned below = (1u << lane) - 1u;
      const int g_me = gt_before + __popc(bgt & below);
      const int e_me = eq_before + __popc(beq & below);
      if (c < hi && (u > T || (u == T && e_me < take_eq))) emit(g_me + min(e_me, take_eq), c);
      gt_before += __popc(bgt);
      eq_before += __popc(beq);
    }
  }
};

// Selection of the r largest of n keys (1 <= r <= n) held in registers:
// thread t holds positions [t*KPT, t*KPT + KPT), positions >= n are ignored.
// Ties go to the lowest position. threshold() histograms the keys relative
// to their minimum in 2048 bins over [min, max] and narrows to the bin that
// holds the r-th largest key, 11 bits per round; compact() emits every
// selected position in ascending order with its rank (#keys > T before it +
// min(#keys == T before it, take_eq)).
template <int NT, int KPT>
struct RegSelect {
  static constexpr int kBins = 2048;
  static constexpr int kRank = 64;  // largest threshold bin ranked pairwise
  static_assert(kBins % NT == 0, "bins per thread");
  uint32_t* hist;   // smem, kBins entries
  int* scratch;     // smem, NT/32 + 8 ints

  HSA_DEV void threshold(const uint32_t (&key)[KPT], int n, int r, uint32_t* T_out, int* take_eq) {
    constexpr int NW = NT / 32, BPT = kBins / NT;
    const int lane = threadIdx.x & 31;
    volatile int* s = scratch + NW + 2;  // [0] min, [1] max, [2] bin, [3] above
    const int p0 = threadIdx.x * KPT;
    // smallest and largest key for which in(key) holds, over the CTA
    auto key_range = [&](auto in, uint32_t* lo_out, uint32_t* hi_out) {
      uint32_t lo = 0xffffffffu, hi = 0u;
#pragma unroll
      for (int j = 0; j < KPT; ++j)
        if (p0 + j < n && in(key[j])) { lo = min(lo, key[j]); hi = max(hi, key[j]); }
      lo = __reduce_min_sync(kFull, lo);
      hi = __reduce_max_sync(kFull, hi);
      if (threadIdx.x == 0) { s[0] = int(0xffffffffu); s[1] = 0; }
      __syncthreads();
      if (lane == 0) { atomicMin((unsigned*)&s[0], lo); atomicMax((unsigned*)&s[1], hi); }
      __syncthreads();
      *lo_out = uint32_t(s[0]);
      *hi_out = uint32_t(s[1]);
      __syncthreads();
    };
    // the bin of `hist` that holds the rem-th largest counted key; rem
    // becomes its rank inside that bin
    auto pick = [&](int& rem) -> uint32_t {
      uint32_t cnt[BPT], tot = 0;
#pragma unroll
      for (int e = 0; e < BPT; ++e) { cnt[e] = hist[threadIdx.x * BPT + e]; tot += cnt[e]; }
      int total;
      const int above = block_exclusive_scan_rev<NT>(int(tot), scratch, &total);
      if (uint32_t(above) < uint32_t(rem) && uint32_t(rem) <= uint32_t(above) + tot) {
        uint32_t a = uint32_t(above);
#pragma unroll
        for (int e = BPT - 1; e >= 0; --e) {
          if (a + cnt[e] >= uint32_t(rem)) { s[2] = threadIdx.x * BPT + e; s[3] = int(a); break; }
          a += cnt[e];
        }
      }
      __syncthreads();
      rem -= s[3];
      return uint32_t(s[2]);
    };
    uint32_t base, kmax;
    key_range([](uint32_t) { return true; }, &base, &kmax);
    int rem = r;
    // First round over bins linear in the score value. Keys are the
    // order-preserving images of fp32 scores; bins on their top bits would
    // crowd a row into the few bins that span its exponents, while linear
    // bins spread it over all of them. The bin floor((x - lo) * c), in
    // round-to-nearest fp32, never decreases as x grows, so every bin is a
    // contiguous key range and the rounds below can continue inside it.
    // Rows whose range is not finite skip this round.
    const float flo = key_score(base), fhi = key_score(kmax);
    const float c = float(kBins) / (fhi - flo);
    if (flo < fhi && c > 0.f && c < INFINITY) {
      auto vbin = [&](uint32_t u) { return min(uint32_t(kBins - 1), __float2uint_rz((key_score(u) - flo) * c)); };
#pragma unroll
      for (int e = 0; e < BPT; ++e) hist[threadIdx.x * BPT + e] = 0;
      __syncthreads();
#pragma unroll
      for (int j = 0; j < KPT; ++j)
        if (p0 + j < n) atomicAdd(&hist[vbin(key[j])], 1u);
      __syncthreads();
      const uint32_t bin = pick(rem);
      const uint32_t cstar = hist[bin];
      const bool whole = cstar == uint32_t(rem);
      if (!whole && cstar <= uint32_t(kRank)) {
        // a bin of at most kRank keys: gather it and rank it pairwise, the
        // rem-th largest of the bin is T
        if (threadIdx.x == 0) s[4] = 0;
        __syncthreads();  // (hist[bin] has been read by every thread)
#pragma unroll
        for (int j = 0; j < KPT; ++j)
          if (p0 + j < n && vbin(key[j]) == bin) hist[atomicAdd((int*)&s[4], 1)] = key[j];
        __syncthreads();
        if (threadIdx.x < int(cstar)) {
          const uint32_t x = hist[threadIdx.x];
          int gt = 0, ge = 0;
          for (int q = 0; q < int(cstar); ++q) {
            const uint32_t y = hist[q];
            gt += y > x;
            ge += y >= x;
          }
          if (gt < rem && rem <= ge) { s[0] = int(x); s[1] = rem - gt; }  // writers agree
        }
        __syncthreads();
        *T_out = uint32_t(s[0]);
        *take_eq = s[1];
        __syncthreads();  // s[] is read before any later use of the scratch
        return;
      }
      key_range([&](uint32_t u) { return vbin(u) == bin; }, &base, &kmax);
      if (whole && base > 0u) {
        *T_out = base - 1u;
        *take_eq = 0;
        return;
      }
    }
    uint32_t width = kmax - base;
    for (;;) {
      const int bits = 32 - __clz(width);
      const int shift = bits > 11 ? bits - 11 : 0;
#pragma unroll
      for (int e = 0; e < BPT; ++e) hist[threadIdx.x * BPT + e] = 0;
      __syncthreads();
#pragma unroll
      for (int j = 0; j < KPT; ++j) {
        const uint32_t d = key[j] - base;
        if (p0 + j < n && d <= width) atomicAdd(&hist[d >> shift], 1u);
      }
      __syncthreads();
      const uint32_t bin = pick(rem);
      const bool whole = hist[bin] == uint32_t(rem);  // every key of the bin is taken
      base += bin << shift;
      width = min(shift ? (1u << shift) - 1u : 0u, kmax - base);
      __syncthreads();
      if (whole && base > 0u) {
        // select every key >= base: threshold just below the bin, no ties taken
        *T_out = base - 1u;
        *take_eq = 0;
        return;
      }
      if (shift == 0) break;
    }
    *T_out = base;
    *take_eq = rem;
  }

  template <class Emit>
  HSA_DEV void compact(const uint32_t (&key)[KPT], int n, uint32_t T, int take_eq, Emit emit) {
    const int p0 = threadIdx.x * KPT;
    int ngt = 0, neq = 0;
#pragma unroll
    for (int j = 0; j < KPT; ++j) {
      ngt += (p0 + j < n && key[j] > T);
      neq += (p0 + j < n && key[j] == T);
    }
    int tot;
    // counts stay below 2^15 per CTA (n <= 16384), so one packed scan serves both
    const int packed = block_exclusive_scan<NT>((ngt << 16) | neq, scratch, &tot);
    int gt = packed >> 16, eq = packed & 0xffff;
#pragma unroll
    for (int j = 0; j < KPT; ++j) {
      if (p0 + j >= n) break;
      if (key[j] > T) {
        emit(gt + min(eq, take_eq), p0 + j);
        ++gt;
      } else if (key[j] == T) {
        if (eq < take_eq) emit(gt + eq, p0 + j);
        ++eq;
      }
    }
  }
};

// Loads keys [p0, p0 + KPT) of row (p0 = threadIdx.x * KPT), 16 bytes at a
// time where the row is 16-byte aligned and complete.
template <int KPT>
HSA_DEV void load_keys(const uint32_t* __restrict__ row, int n, uint32_t (&key)[KPT]) {
  const int p0 = threadIdx.x * KPT;
  if constexpr (KPT % 4 == 0) {
    if (p0 + KPT <= n && (reinterpret_cast<uintptr_t>(row) & 15u) == 0) {
#pragma unroll
      for (int v = 0; v < KPT / 4; ++v) {
        const uint4 q = __ldg(reinterpret_cast<const uint4*>(row + p0) + v);
        key[4 * v] = q.x; key[4 * v + 1] = q.y; key[4 * v + 2] = q.z; key[4 * v + 3] = q.w;
      }
      return;
    }
  }
#pragma unroll
  for (int j = 0; j < KPT; ++j) key[j] = p0 + j < n ? __ldg(row + p0 + j) : 0u;
}

}  // namespace hsa
