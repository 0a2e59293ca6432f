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
HSA_DEV uint32_t pack_bf16x2(float lo, float hi) {
  return f32_to_bf16_rn(lo) | (f32_to_bf16_rn(hi) << 16);
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

// CTA-wide selection of the r largest of n keys (1 <= r <= n), ties broken
// towards the lowest position. MSB-first radix search with 8-bit digits over
// the 32-bit keys finds the r-th largest key T; every key > T is taken and,
// of the keys == T, the `take_eq` at the lowest positions.
template <int NT>
struct RadixSelect {
  uint32_t* hist;   // smem, 256 entries
  int* scratch;     // smem, NT/32 + 8 ints

  HSA_DEV void threshold(const uint32_t* keys, int n, int r, uint32_t* T_out, int* take_eq) {
    uint32_t prefix = 0, mask = 0;
    int rem = r;
    volatile int* s_res = scratch + NT / 32 + 2;  // [digit, above]
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (int e = threadIdx.x; e < 256; e += NT) hist[e] = 0;
      __syncthreads();
      for (int c = threadIdx.x; c < n; c += NT) {
        uint32_t u = keys[c];
        if ((u & mask) == prefix) atomicAdd(&hist[(u >> shift) & 255u], 1u);
      }
      __syncthreads();
      if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        uint32_t c8[8], tot = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) { c8[e] = hist[lane * 8 + e]; tot += c8[e]; }
        uint32_t incl = tot;  // sum over lanes >= lane
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          uint32_t y = __shfl_down_sync(kFull, incl, o);
          if (lane + o < 32) incl += y;
        }
        const uint32_t above = incl - tot;
        if (above < uint32_t(rem) && uint32_t(rem) <= incl) {
          uint32_t a = above;
          for (int e = 7; e >= 0; --e) {
            if (a + c8[e] >= uint32_t(rem)) { s_res[0] = lane * 8 + e; s_res[1] = int(a); break; }
            a += c8[e];
          }
        }
      }
      __syncthreads();
      const uint32_t digit = uint32_t(s_res[0]);
      rem -= s_res[1];
      prefix |= digit << shift;
      mask |= 255u << shift;
      __syncthreads();
    }
    *T_out = prefix;
    *take_eq = rem;
  }

  // Writes the positions of the selected keys, ascending, via emit(rank, pos).
  // Warps own contiguous position ranges; lanes interleave inside them.
  template <class Emit>
  HSA_DEV void compact(const uint32_t* keys, int n, uint32_t T, int take_eq, Emit emit) {
    constexpr int NW = NT / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int per = ((n + NW * 32 - 1) / (NW * 32)) * 32;
    const int lo = warp * per, hi = min(n, lo + per);
    int neq = 0;
    for (int c0 = lo; c0 < hi; c0 += 32) {
      const int c = c0 + lane;
      neq += __popc(__ballot_sync(kFull, c < hi && keys[c] == T));
    }
    int tot;
    int eq_before = block_exclusive_scan<NT>(lane == 0 ? neq : 0, scratch, &tot);
    eq_before = __shfl_sync(kFull, eq_before, 0);
    int nsel = 0, eqs = eq_before;
    for (int c0 = lo; c0 < hi; c0 += 32) {
      const int c = c0 + lane;
      const uint32_t u = c < hi ? keys[c] : 0u;
      const unsigned beq = __ballot_sync(kFull, c < hi && u == T);
      const int my_eq_rank = eqs + __popc(beq & ((1u << lane) - 1u));
      const bool sel = c < hi && (u > T || (u == T && my_eq_rank < take_eq));
      nsel += __popc(__ballot_sync(kFull, sel));
      eqs += __popc(beq);
    }
    int sel_before = block_exclusive_scan<NT>(lane == 0 ? nsel : 0, scratch, &tot);
    sel_before = __shfl_sync(kFull, sel_before, 0);
    eqs = eq_before;
    int out = sel_before;
    for (int c0 = lo; c0 < hi; c0 += 32) {
      const int c = c0 + lane;
      const uint32_t u = c < hi ? keys[c] : 0u;
      const unsigned beq = __ballot_sync(kFull, c < hi && u == T);
      const int my_eq_rank = eqs + __popc(beq & ((1u << lane) - 1u));
      const bool sel = c < hi && (u > T || (u == T && my_eq_rank < take_eq));
      const unsigned bs = __ballot_sync(kFull, sel);
      if (sel) emit(out + __popc(bs & ((1u << lane) - 1u)), c);
      out += __popc(bs);
      eqs += __popc(beq);
    }
  }
};

}  // namespace hsa
