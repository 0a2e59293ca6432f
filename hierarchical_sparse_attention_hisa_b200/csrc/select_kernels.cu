// Selections over scores produced by the tensor-core scoring kernels, and
// the per-block work lists that feed the token-scoring GEMM.
//
//   top-m blocks   (section 第一步 + the forced first/last block note): from
//                  the block-score keys of one query row;
//   pair lists     every (query row, slot) whose kept block b still needs
//                  token scores, grouped by b into tiles of <= 128 pairs;
//   top-k tokens   (section 第二步): from the token-score keys of one row,
//                  candidates enumerated in ascending token order.
#include "kernels.cuh"
#include "tc.cuh"

namespace hsa {
namespace {

constexpr int NT = 256;
constexpr int kMaxRowBlocks = 512;  // kept blocks per row the selections hold in shared memory

// Kept-block list of one row: count of valid entries and candidate count
// (tokens j <= t of the kept blocks). Returns false when the list does not
// have the selector's shape (ascending, the query's own block last).
HSA_DEV bool row_candidates(const int32_t* blk, int m, int64_t t, int B, int* nblk_out, int* ncand_out) {
  int nblk = 0;
  while (nblk < m && blk[nblk] >= 0) ++nblk;
  if (nblk == 0 || blk[nblk - 1] != int(t / B)) return false;
  for (int s = 0; s + 1 < nblk; ++s)
    if (blk[s] >= blk[s + 1]) return false;
  *nblk_out = nblk;
  *ncand_out = int((nblk - 1) * int64_t(B) + (t - int64_t(blk[nblk - 1]) * B + 1));
  return true;
}

// The same check by the 32 lanes of a warp together (every lane gets the
// result): lane l reads entries l, l + 32, ... of the list.
HSA_DEV bool warp_row_candidates(const int32_t* blk, int m, int64_t t, int B, int* nblk_out, int* ncand_out) {
  const int lane = threadIdx.x & 31;
  int nblk = m;
  for (int s0 = 0; s0 < m && nblk == m; s0 += 32) {
    const int s = s0 + lane;
    const unsigned neg = __ballot_sync(kFull, s < m && blk[s] < 0);
    if (neg) nblk = s0 + __ffs(neg) - 1;
  }
  if (nblk == 0) return false;  // (warp-uniform)
  bool ok = true;
  for (int s = lane; s + 1 < nblk; s += 32) ok = ok && blk[s] < blk[s + 1];
  ok = __all_sync(kFull, ok) && blk[nblk - 1] == int(t / B);
  *nblk_out = nblk;
  *ncand_out = int((nblk - 1) * int64_t(B) + (t - int64_t(blk[nblk - 1]) * B + 1));
  return ok;
}

// Keys of positions [p0, p0 + KPT) of the row that starts one key after
// `row` (p0 = threadIdx.x * KPT), positions >= n read as 0: from 16-byte
// loads of `row` itself (aligned) shifted by one key, where the row (of ld
// keys) holds them all, else one key at a time.
template <int KPT>
HSA_DEV void load_keys_after_first(const uint32_t* __restrict__ row, int64_t ld, int n, uint32_t (&key)[KPT]) {
  const int p0 = threadIdx.x * KPT;
  if constexpr (KPT % 4 == 0) {
    if (p0 + KPT <= n && p0 + KPT + 4 <= ld && (reinterpret_cast<uintptr_t>(row) & 15u) == 0) {
      uint32_t v[KPT + 4];
#pragma unroll
      for (int q = 0; q < KPT / 4 + 1; ++q) {
        const uint4 x = __ldg(reinterpret_cast<const uint4*>(row + p0) + q);
        v[4 * q] = x.x; v[4 * q + 1] = x.y; v[4 * q + 2] = x.z; v[4 * q + 3] = x.w;
      }
#pragma unroll
      for (int j = 0; j < KPT; ++j) key[j] = v[j + 1];
      return;
    }
  }
#pragma unroll
  for (int j = 0; j < KPT; ++j) key[j] = p0 + j < n ? __ldg(row + 1 + p0 + j) : 0u;
}

template <int KPT>
__global__ void __launch_bounds__(NT, 3) topm_from_keys_kernel(RowMap rm, const uint32_t* __restrict__ bkeys,
                                                           int64_t ld, int B, int m, int32_t* __restrict__ blocks) {
  griddep_wait();
  griddep_launch();
  __shared__ uint32_t hist[RegSelect<NT, KPT>::kBins];
  __shared__ int scratch[NT / 32 + 8];
  const int64_t i = blockIdx.x;
  int32_t* out = blocks + i * m;
  if (!rm.valid(i)) {
    for (int s = threadIdx.x; s < m; s += NT) out[s] = -1;
    return;
  }
  const int64_t t = rm.pos(i);
  const int64_t nb = t / B + 1;
  if (nb <= m) {
    for (int s = threadIdx.x; s < m; s += NT) out[s] = s < nb ? s : -1;
    return;
  }
  if (m == 2) {
    if (threadIdx.x == 0) { out[0] = 0; out[1] = int32_t(nb - 1); }
    return;
  }
  const int n = int(nb - 2);  // candidates: blocks 1 .. nb-2
  uint32_t key[KPT];
  load_keys_after_first<KPT>(bkeys + i * ld, ld, n, key);
  RegSelect<NT, KPT> rs{hist, scratch};
  uint32_t T;
  int take_eq;
  rs.threshold(key, n, m - 2, &T, &take_eq);
  if (threadIdx.x == 0) { out[0] = 0; out[m - 1] = int32_t(nb - 1); }
  rs.compact(key, n, T, take_eq, [&](int rank, int c) { out[1 + rank] = c + 1; });
}

// Top-m with one warp per row, for rows of at most 32 * KPT candidate blocks
// (many rows, few candidates each: no CTA barriers). Lane l holds the keys of
// candidates e * 32 + l. The threshold T, the (m-2)-th largest key, is found
// in a warp-private histogram: one pass over bins linear in the score and a
// direct ranking of the threshold bin's keys, or, when that bin is crowded,
// radix selection 8 key bits a pass from the top. Selected candidates are
// written in ascending order, ties at T going to the lowest positions,
// exactly as the block-wide selection.
constexpr int kTopmWarpsPerCta = 8;

template <int KPT>
__global__ void __launch_bounds__(32 * kTopmWarpsPerCta) topm_warp_rows_kernel(
    RowMap rm, int64_t rows, const uint32_t* __restrict__ bkeys, int64_t ld, int B, int m,
    int32_t* __restrict__ blocks) {
  griddep_wait();
  griddep_launch();
  const int lane = threadIdx.x & 31;
  const int64_t i = int64_t(blockIdx.x) * kTopmWarpsPerCta + (threadIdx.x >> 5);
  if (i >= rows) return;
  int32_t* out = blocks + i * m;
  if (!rm.valid(i)) {
    for (int s = lane; s < m; s += 32) out[s] = -1;
    return;
  }
  const int64_t t = rm.pos(i);
  const int64_t nb = t / B + 1;
  if (nb <= m) {
    for (int s = lane; s < m; s += 32) out[s] = s < nb ? s : -1;
    return;
  }
  if (m == 2) {
    if (lane == 0) { out[0] = 0; out[1] = int32_t(nb - 1); }
    return;
  }
  const int n = int(nb - 2);  // candidates: blocks 1 .. nb-2
  const int r = m - 2;
  const uint32_t* src = bkeys + i * ld + 1;
  uint32_t key[KPT];
#pragma unroll
  for (int e = 0; e < KPT; ++e) key[e] = e * 32 + lane < n ? __ldg(src + e * 32 + lane) : 0u;
  __shared__ __align__(16) uint32_t whist[kTopmWarpsPerCta][256];
  __shared__ uint32_t wlist[kTopmWarpsPerCta][32];
  uint32_t* hist = whist[threadIdx.x >> 5];
  auto clear_hist = [&]() {
    reinterpret_cast<uint4*>(hist)[2 * lane] = make_uint4(0, 0, 0, 0);
    reinterpret_cast<uint4*>(hist)[2 * lane + 1] = make_uint4(0, 0, 0, 0);
  };
  // the bin of the histogram holding the rem-th largest counted key; rem
  // becomes the rank inside it (lane l holds bins 8l .. 8l+7)
  auto pick = [&](int& rem) -> int {
    uint32_t cnt[8], tot = 0;
#pragma unroll
    for (int q = 0; q < 8; ++q) { cnt[q] = hist[lane * 8 + q]; tot += cnt[q]; }
    uint32_t suf = tot;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_down_sync(kFull, suf, o);
      if (lane + o < 32) suf += y;
    }
    const uint32_t above = suf - tot;
    const bool holds = above < uint32_t(rem) && uint32_t(rem) <= above + tot;
    int dsel = 0, nrem = 0;
    if (holds) {
      uint32_t acc = above;
#pragma unroll
      for (int q = 7; q >= 0; --q) {
        if (dsel == 0 && nrem == 0 && acc + cnt[q] >= uint32_t(rem)) { dsel = lane * 8 + q; nrem = rem - int(acc); }
        acc += cnt[q];
      }
    }
    const int from = __ffs(__ballot_sync(kFull, holds)) - 1;
    rem = __shfl_sync(kFull, nrem, from);
    return __shfl_sync(kFull, dsel, from);
  };
  // The (m-2)-th largest key T. First in 256 bins linear in the score (see
  // the top-k rows): the threshold bin usually holds a few keys, which are
  // ranked directly. Otherwise radix selection on the key bits, 8 bits a pass
  // from the top (lanes holding the same digit add once, through a match).
  uint32_t T = 0;
  int take_eq = -1;
  {
    uint32_t lo = 0xffffffffu, hi = 0u;
#pragma unroll
    for (int e = 0; e < KPT; ++e)
      if (e * 32 + lane < n) { lo = min(lo, key[e]); hi = max(hi, key[e]); }
    lo = __reduce_min_sync(kFull, lo);
    hi = __reduce_max_sync(kFull, hi);
    const float flo = key_score(lo), fhi = key_score(hi);
    const float c = 253.0f / (fhi - flo);
    if (flo < fhi && c > 0.f && c < INFINITY) {
      const float nb = 12582913.0f - flo * c;  // bin = (x - lo) * c + 1, rounded
      auto bin_of = [&](uint32_t u) {
        return min(255, max(0, int(__float_as_uint(fmaf(key_score(u), c, nb)) - 0x4B400000u)));
      };
      clear_hist();
      __syncwarp();
#pragma unroll
      for (int e = 0; e < KPT; ++e)
        if (e * 32 + lane < n) atomicAdd(&hist[bin_of(key[e])], 1u);
      __syncwarp();
      int rem = r;
      const int bsel = pick(rem);
      const uint32_t cstar = hist[bsel];
      if (cstar <= 32u) {
        // gather the threshold bin and rank its keys pairwise
        int cnt = 0;
#pragma unroll
        for (int e = 0; e < KPT; ++e) {
          const bool in = e * 32 + lane < n && bin_of(key[e]) == bsel;
          const unsigned bi = __ballot_sync(kFull, in);
          if (in) wlist[threadIdx.x >> 5][cnt + __popc(bi & ((1u << lane) - 1u))] = key[e];
          cnt += __popc(bi);
        }
        __syncwarp();
        int gt = 0, ge = 0;
        const uint32_t x = lane < int(cstar) ? wlist[threadIdx.x >> 5][lane] : 0u;
        for (int q = 0; q < int(cstar); ++q) {
          const uint32_t y = wlist[threadIdx.x >> 5][q];
          gt += y > x;
          ge += y >= x;
        }
        const bool hit = lane < int(cstar) && gt < rem && rem <= ge;
        const int from = __ffs(__ballot_sync(kFull, hit)) - 1;
        T = __shfl_sync(kFull, x, from);
        take_eq = __shfl_sync(kFull, rem - gt, from);
      }
      __syncwarp();  // every lane has read the histogram before it is cleared
    }
  }
  if (take_eq < 0) {
    uint32_t tmask = 0;
    int rem = r;  // rank of T among the keys that share the digits chosen so far
    for (int shift = 24; shift >= 0; shift -= 8) {
      clear_hist();
      __syncwarp();
#pragma unroll
      for (int e = 0; e < KPT; ++e) {
        const bool in = e * 32 + lane < n && (key[e] & tmask) == T;
        const uint32_t d = in ? (key[e] >> shift) & 255u : 256u;
        const unsigned same = __match_any_sync(kFull, d);
        if (in && lane == __ffs(same) - 1) atomicAdd(&hist[d], uint32_t(__popc(same)));
      }
      __syncwarp();
      const int dsel = pick(rem);
      T |= uint32_t(dsel) << shift;
      tmask |= 255u << shift;
      __syncwarp();  // every lane has read the histogram before it is cleared
    }
    take_eq = rem;
  }
  if (lane == 0) { out[0] = 0; out[m - 1] = int32_t(nb - 1); }
  const unsigned below = (1u << lane) - 1u;
  int base = 0, eqb = 0;
#pragma unroll
  for (int e = 0; e < KPT; ++e) {
    const int c = e * 32 + lane;
    const bool live = c < n;
    const bool gt = live && key[e] > T, eq = live && key[e] == T;
    const unsigned beq = __ballot_sync(kFull, eq);
    const bool take = gt || (eq && eqb + __popc(beq & below) < take_eq);
    const unsigned bt = __ballot_sync(kFull, take);
    if (take) out[1 + base + __popc(bt & below)] = c + 1;
    base += __popc(bt);
    eqb += __popc(beq);
  }
}

// Pairs of the rows [r0, r0 + ROWS) that need token scores, binned by block.
// The scatter pass also writes the tile table: CTA c the tiles (block, first
// pair, pair count) of bins c, c + gridDim.x, ...
constexpr int kPairRows = 64;  // rows per CTA, fewer when that leaves SMs idle

template <bool SCATTER>
__global__ void __launch_bounds__(NT) pair_bin_kernel(RowMap rm, int64_t rows, const int32_t* __restrict__ blocks,
                                                     int B, int m, int k, int nbins, int rows_per_cta,
                                                     int* __restrict__ cnt,
                                                     const int* __restrict__ off, int* __restrict__ cursor,
                                                     uint32_t* __restrict__ pairs, int4* __restrict__ tiles) {
  griddep_wait();
  griddep_launch();
  extern __shared__ int sh[];
  int* hist = sh;             // [nbins]
  int* base = sh + nbins;     // [nbins] (scatter only)
  for (int b = threadIdx.x; b < nbins; b += NT) hist[b] = 0;
  __syncthreads();
  const int64_t r0 = int64_t(blockIdx.x) * rows_per_cta;
  // one warp per row at a time; lanes over slots
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto row_pairs = [&](auto&& fn) {
    for (int rr = warp; rr < rows_per_cta; rr += NT / 32) {
      const int64_t i = r0 + rr;
      if (i >= rows) break;
      const int32_t* blk = blocks + i * m;
      const int64_t t = rm.pos(i);
      int nblk = 0, ncand = 0;
      if (!warp_row_candidates(blk, m, t, B, &nblk, &ncand) || ncand <= k) continue;
      for (int s = lane; s < nblk; s += 32) fn(i, s, blk[s]);
    }
  };
  row_pairs([&](int64_t, int, int b) { atomicAdd(&hist[b], 1); });
  __syncthreads();
  if (!SCATTER) {
    for (int b = threadIdx.x; b < nbins; b += NT)
      if (hist[b]) atomicAdd(&cnt[b], hist[b]);
    return;
  }
  for (int b = threadIdx.x; b < nbins; b += NT) {
    base[b] = hist[b] ? off[b] + atomicAdd(&cursor[b], hist[b]) : 0;
    hist[b] = 0;
  }
  for (int b = blockIdx.x; b < nbins; b += gridDim.x) {
    const int c = cnt[b], o = off[b], to = off[nbins + b];
    for (int u = threadIdx.x; 128 * u < c; u += NT) tiles[to + u] = make_int4(b, o + 128 * u, min(128, c - 128 * u), 0);
  }
  __syncthreads();
  row_pairs([&](int64_t i, int s, int b) {
    const int pos = base[b] + atomicAdd(&hist[b], 1);
    pairs[pos] = uint32_t(i) * uint32_t(m) + uint32_t(s);
  });
}

// Single CTA: each bin's first pair (off[b]) and first tile (off[nbins + b])
// in tiles of <= 128 pairs, and the tile count.
__global__ void __launch_bounds__(1024) pair_scan_kernel(int nbins, const int* __restrict__ cnt, int* __restrict__ off,
                                                        int* __restrict__ cursor, int* __restrict__ ntiles) {
  griddep_wait();
  griddep_launch();
  __shared__ int s_tmp[1024 / 32 + 1];
  __shared__ int carry_pairs, carry_tiles;
  if (threadIdx.x == 0) { carry_pairs = 0; carry_tiles = 0; }
  __syncthreads();
  for (int b0 = 0; b0 < nbins; b0 += 1024) {
    const int b = b0 + threadIdx.x;
    const int c = b < nbins ? cnt[b] : 0;
    const int nt = (c + 127) / 128;
    int tot_p, tot_t;
    const int ep = block_exclusive_scan<1024>(c, s_tmp, &tot_p);
    const int et = block_exclusive_scan<1024>(nt, s_tmp, &tot_t);
    if (b < nbins) {
      off[b] = carry_pairs + ep;
      off[nbins + b] = carry_tiles + et;
      cursor[b] = 0;
    }
    __syncthreads();
    if (threadIdx.x == 0) { carry_pairs += tot_p; carry_tiles += tot_t; }
    __syncthreads();
  }
  if (threadIdx.x == 0) *ntiles = carry_tiles;
}

template <int NT, int KPT>
__global__ void __launch_bounds__(NT) topk_from_keys_kernel(RowMap rm, const int32_t* __restrict__ blocks,
                                                           const uint32_t* __restrict__ tkeys, int B, int m,
                                                           int k, int32_t* __restrict__ indices) {
  griddep_wait();
  griddep_launch();
  __shared__ uint32_t hist[RegSelect<NT, KPT>::kBins];
  __shared__ int scratch[NT / 32 + 8];
  __shared__ int blk[kMaxRowBlocks];
  __shared__ int s_info[3];
  const int64_t i = blockIdx.x;
  int32_t* out = indices + i * int64_t(k);
  if (!rm.valid(i)) {
    for (int s = threadIdx.x; s < k; s += NT) out[s] = -1;
    return;
  }
  const int64_t t = rm.pos(i);
  for (int s = threadIdx.x; s < m; s += NT) blk[s] = blocks[i * m + s];
  __syncthreads();
  if (threadIdx.x == 0) {
    int nblk = 0, ncand = 0;
    s_info[0] = row_candidates(blk, m, t, B, &nblk, &ncand);
    s_info[1] = nblk;
    s_info[2] = ncand;
  }
  __syncthreads();
  if (!s_info[0]) {
    for (int s = threadIdx.x; s < k; s += NT) out[s] = -1;
    return;
  }
  const int n = s_info[2];
  const bool pow2 = (B & (B - 1)) == 0;
  const int lb = 31 - __clz(B);
  auto tok = [&](int c) -> int32_t {
    return pow2 ? (blk[c >> lb] << lb) + (c & (B - 1)) : int32_t(int64_t(blk[c / B]) * B + c % B);
  };
  if (n <= k) {
    for (int s = threadIdx.x; s < k; s += NT) out[s] = s < n ? tok(s) : -1;
    return;
  }
  uint32_t key[KPT];
  load_keys<KPT>(tkeys + i * int64_t(m) * B, n, key);
  RegSelect<NT, KPT> rs{hist, scratch};
  uint32_t T;
  int take_eq;
  rs.threshold(key, n, k, &T, &take_eq);
  rs.compact(key, n, T, take_eq, [&](int rank, int c) { out[rank] = tok(c); });
}

// ---------------------------------------------------------------------------
// Top-k with one warp per row (many rows): no CTA barriers. The warp streams
// its row's keys (16-byte loads) once for min/max, once per 11-bit histogram
// round into a warp-private 2048-bin shared histogram, and once to emit the
// selected positions in ascending order.
// ---------------------------------------------------------------------------
constexpr int kWarpRowsPerCta = 8;
constexpr int kWBins = 2048;

// Calls f(key) for the keys [0, n) of `row`: 16-byte loads, lane-strided,
// two 128-key steps in flight per iteration, scalar loads for the tail.
template <class F>
HSA_DEV void warp_stream_keys(const uint32_t* __restrict__ row, int n, F f) {
  const int lane = threadIdx.x & 31;
  const int n8 = n & ~255, n4 = n & ~127;
  const uint4* r4 = reinterpret_cast<const uint4*>(row);
  for (int c0 = 0; c0 < n8; c0 += 256) {
    const uint4 a = __ldg(r4 + (c0 >> 2) + lane), b = __ldg(r4 + (c0 >> 2) + 32 + lane);
    f(a.x); f(a.y); f(a.z); f(a.w); f(b.x); f(b.y); f(b.z); f(b.w);
  }
  if (n4 > n8) {
    const uint4 a = __ldg(r4 + (n8 >> 2) + lane);
    f(a.x); f(a.y); f(a.z); f(a.w);
  }
  for (int c = n4 + lane; c < n; c += 32) f(__ldg(row + c));
}

__global__ void __launch_bounds__(32 * kWarpRowsPerCta) topk_warp_rows_kernel(
    RowMap rm, int64_t rows, const int32_t* __restrict__ blocks, const uint32_t* __restrict__ tkeys, int B,
    int m, int k, int32_t* __restrict__ indices) {
  extern __shared__ uint32_t wsm[];  // per warp: kWBins histogram bins, then kMaxRowBlocks block ids
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t i = int64_t(blockIdx.x) * kWarpRowsPerCta + warp;
  if (i >= rows) return;
  uint32_t* hist = wsm + warp * (kWBins + kMaxRowBlocks);
  int* blk = reinterpret_cast<int*>(hist + kWBins);
  int32_t* out = indices + i * int64_t(k);
  if (!rm.valid(i)) {
    for (int s = lane; s < k; s += 32) out[s] = -1;
    return;
  }
  const int64_t t = rm.pos(i);
  for (int s = lane; s < m; s += 32) blk[s] = blocks[i * m + s];
  __syncwarp();
  int nblk = 0, n = 0;
  const bool ok = warp_row_candidates(blk, m, t, B, &nblk, &n);
  if (!ok) {
    for (int s = lane; s < k; s += 32) out[s] = -1;
    return;
  }
  const bool pow2 = (B & (B - 1)) == 0;
  const int lb = 31 - __clz(B);
  auto tok = [&](int c) -> int32_t {
    return pow2 ? (blk[c >> lb] << lb) + (c & (B - 1)) : int32_t(int64_t(blk[c / B]) * B + c % B);
  };
  if (n <= k) {
    for (int s = lane; s < k; s += 32) out[s] = s < n ? tok(s) : -1;
    return;
  }
  const uint32_t* row = tkeys + i * int64_t(m) * B;
  // narrow to the k-th largest key, 11 bits per round from the top
  // (rounds of 11, 11 and 10 bits; a bin taken whole ends the search early)
  const uint32_t hi = 0xffffffffu;
  uint32_t base = 0u, width = 0xffffffffu, T = 0;
  int rem = k, take_eq = 0;
  for (;;) {
    const int bits = 32 - __clz(width);
    const int shift = bits > 11 ? bits - 11 : 0;
    for (int e = lane; e < kWBins; e += 32) hist[e] = 0;
    __syncwarp();
    warp_stream_keys(row, n, [&](uint32_t u) {
      const uint32_t d = u - base;
      if (d <= width) atomicAdd(&hist[d >> shift], 1u);
    });
    __syncwarp();
    // lane l owns bins [64 l, 64 l + 64); counts above each lane's range
    uint32_t tot = 0;
    for (int e = 0; e < 64; ++e) tot += hist[lane * 64 + e];
    uint32_t incl = tot;  // sum over lanes >= lane
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_down_sync(kFull, incl, o);
      if (lane + o < 32) incl += y;
    }
    const uint32_t above = incl - tot;
    int found_bin = -1;
    uint32_t found_above = 0;
    if (above < uint32_t(rem) && uint32_t(rem) <= incl) {
      uint32_t a = above;
      for (int e = 63; e >= 0; --e) {
        const uint32_t c = hist[lane * 64 + e];
        if (a + c >= uint32_t(rem)) { found_bin = lane * 64 + e; found_above = a; break; }
        a += c;
      }
    }
    const unsigned who = __ballot_sync(kFull, found_bin >= 0);
    const int src = __ffs(who) - 1;
    const uint32_t bin = uint32_t(__shfl_sync(kFull, found_bin, src));
    rem -= int(__shfl_sync(kFull, found_above, src));
    const bool whole = hist[bin] == uint32_t(rem);
    base += bin << shift;
    width = min(shift ? (1u << shift) - 1u : 0u, hi - base);
    __syncwarp();
    if (whole && base > 0u) { T = base - 1u; take_eq = 0; break; }
    if (shift == 0) { T = base; take_eq = rem; break; }
  }
  // emit ascending: rank = (#keys > T before) + min(#keys == T before, take_eq)
  int gt = 0, eq = 0;
  const int n4 = n & ~127;
  const unsigned below = (1u << lane) - 1u;
  for (int c0 = 0; c0 < n4; c0 += 128) {
    const int c = c0 + 4 * lane;
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(row + c));
    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
    int g4 = 0, e4 = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) { g4 += u[e] > T; e4 += u[e] == T; }
    // exclusive prefix of the lane counts
    int gp = g4, ep = e4;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int yg = __shfl_up_sync(kFull, gp, o), ye = __shfl_up_sync(kFull, ep, o);
      if (lane >= o) { gp += yg; ep += ye; }
    }
    int gb = gt + gp - g4, eb = eq + ep - e4;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (u[e] > T) { out[gb + min(eb, take_eq)] = tok(c + e); ++gb; }
      else if (u[e] == T) { if (eb < take_eq) out[gb + eb] = tok(c + e); ++eb; }
    }
    gt += __shfl_sync(kFull, gp, 31);
    eq += __shfl_sync(kFull, ep, 31);
  }
  for (int c0 = n4; c0 < n; c0 += 32) {
    const int c = c0 + lane;
    const uint32_t u = c < n ? __ldg(row + c) : 0u;
    const unsigned bg = __ballot_sync(kFull, c < n && u > T);
    const unsigned be = __ballot_sync(kFull, c < n && u == T);
    const int gb = gt + __popc(bg & below), eb = eq + __popc(be & below);
    if (c < n && u > T) out[gb + min(eb, take_eq)] = tok(c);
    else if (c < n && u == T && eb < take_eq) out[gb + eb] = tok(c);
    gt += __popc(bg);
    eq += __popc(be);
  }
  (void)nblk;
}

// One row per 256-thread CTA (m*B <= 8192, B a power of two >= 4): the row's keys
// are staged once in shared memory and every pass reads them from there.
// Thread t owns positions [32 t, 32 t + 32) as eight 16-byte chunks whose
// slots are XOR-swizzled, so that the coalesced fill and a warp reading one
// chunk of each of its threads are both free of bank conflicts.
// The threshold is located first in 2048 bins linear in the score value
// (bins on key bits would crowd a row into the few bins of its exponent
// range). The bin function never decreases as the score grows, so a bin is a
// contiguous key range; it usually holds a handful of keys, which are
// gathered and ranked directly. A crowded bin, or a row whose score range is
// not finite, continues with 11-bit rounds on the key bits. The k selected
// indices are assembled in shared memory and leave with coalesced stores.
constexpr int kRowNT = 256, kRowCap = 8192, kRowKPT = kRowCap / kRowNT, kRowChunks = kRowKPT / 4;
constexpr int kRowBins = 2048, kRowBPT = kRowBins / kRowNT;
constexpr int kRowRank = 64;  // largest threshold bin ranked pairwise
static_assert(kRowChunks == 8, "chunk swizzle assumes eight chunks per thread");

struct RowSmem {
  uint4 keys[kRowCap / 4];
  uint32_t hist[kRowBins];
  uint32_t list[kRowRank];
  int blk[256];
  int sc[16];
  uint32_t red[32];  // [0..7] minima, [8..15] maxima, [16] list count, [17] T, [18] take_eq, [19..20] bin range
  int pk[2];
};

// Bits 0..15 of x to the even positions, bits 16..31 to the odd ones.
HSA_DEV uint32_t interleave_halves(uint32_t x) {
  uint32_t t = (x ^ (x >> 8)) & 0x0000ff00u;
  x ^= t ^ (t << 8);
  t = (x ^ (x >> 4)) & 0x00f000f0u;
  x ^= t ^ (t << 4);
  t = (x ^ (x >> 2)) & 0x0c0c0c0cu;
  x ^= t ^ (t << 2);
  t = (x ^ (x >> 1)) & 0x22222222u;
  x ^= t ^ (t << 1);
  return x;
}

HSA_DEV int row_slot(int g) { return (g & ~7) | ((g & 7) ^ ((g >> 3) & 7)); }

__global__ void __launch_bounds__(kRowNT, 5) topk_rows_kernel(RowMap rm, const int32_t* __restrict__ blocks,
                                                           const uint32_t* __restrict__ tkeys, int B, int m,
                                                           int k, int32_t* __restrict__ indices) {
  griddep_wait();
  griddep_launch();
  extern __shared__ __align__(16) uint8_t row_smem_raw[];
  RowSmem& S = *reinterpret_cast<RowSmem*>(row_smem_raw);
  const int tid = threadIdx.x, w = tid >> 5, l = tid & 31;
  const int64_t i = blockIdx.x;
  int32_t* out = indices + i * int64_t(k);
  if (!rm.valid(i)) {
    for (int s = tid; s < k; s += kRowNT) out[s] = -1;
    return;
  }
  const int64_t t = rm.pos(i);
  // stage the row's key slots first (every candidate and the unused tail);
  // warp 0 checks the kept-block list while they land
  {
    // slot g = tid + kRowNT * u lands at row_slot(tid) + kRowNT * u (the
    // swizzle only mixes bits below kRowNT)
    const int nslot4 = (m * B) >> 2;
    const uint4* src = reinterpret_cast<const uint4*>(tkeys + i * int64_t(m) * B) + tid;
    const uint32_t dst = tc::smem_u32(&S.keys[row_slot(tid)]);
#pragma unroll
    for (int u = 0; u < kRowCap / 4 / kRowNT; ++u)
      if (tid + u * kRowNT < nslot4) tc::cp_async16(dst + u * kRowNT * 16, src + u * kRowNT);
  }
  for (int e = 0; e < kRowBPT; ++e) S.hist[tid * kRowBPT + e] = 0;
  if (w == 0) {
    // leading entries >= 0 (nblk of them), ascending, the query's own block last
    int nblk = m;
    for (int s0 = 0; s0 < m; s0 += 32) {
      const int s = s0 + l;
      const int bk = s < m ? blocks[i * m + s] : -1;
      if (s < m) S.blk[s] = bk;
      const unsigned neg = __ballot_sync(kFull, s < m && bk < 0);
      if (neg && nblk == m) nblk = s0 + __ffs(neg) - 1;
    }
    __syncwarp();
    bool ordered = true;
    for (int s = l; s + 1 < nblk; s += 32) ordered = ordered && S.blk[s] < S.blk[s + 1];
    ordered = __all_sync(kFull, ordered);
    if (l == 0) {
      const bool ok = ordered && nblk > 0 && S.blk[nblk - 1] == int(t / B);
      S.pk[0] = ok ? int((nblk - 1) * int64_t(B) + (t - int64_t(S.blk[nblk - 1]) * B + 1)) : -1;
      S.red[16] = 0;
    }
  }
  tc::cp_async_wait_all();
  __syncthreads();
  const int n = S.pk[0];
  if (n < 0) {
    for (int s = tid; s < k; s += kRowNT) out[s] = -1;
    return;
  }
  const int lb = 31 - __clz(B);  // B is a power of two here
  if (n <= k) {
    for (int s = tid; s < k; s += kRowNT) out[s] = s < n ? (S.blk[s >> lb] << lb) + (s & (B - 1)) : -1;
    return;
  }
  const int p0 = tid * kRowKPT;
  const int nj = max(0, min(kRowKPT, n - p0));  // this thread's candidates: keys j < nj
  const uint32_t jmask = nj >= 32 ? 0xffffffffu : (1u << nj) - 1u;
  auto chunk = [&](int c) { return S.keys[(tid << 3) | (c ^ (tid & 7))]; };
  auto key_at = [&](int j) {
    const uint4 v = chunk(j >> 2);
    return (j & 3) == 0 ? v.x : (j & 3) == 1 ? v.y : (j & 3) == 2 ? v.z : v.w;
  };
  // f(j, key) for all 32 keys of this thread (fully unrolled: j is a
  // constant); f must ignore j >= nj
  auto each = [&](auto f) {
#pragma unroll
    for (int c = 0; c < kRowChunks; ++c) {
      const uint4 v = chunk(c);
      f(4 * c, v.x);
      f(4 * c + 1, v.y);
      f(4 * c + 2, v.z);
      f(4 * c + 3, v.w);
    }
  };
  auto block_min_max = [&](uint32_t lo, uint32_t hi, uint32_t* lo_out, uint32_t* hi_out) {
    lo = __reduce_min_sync(kFull, lo);
    hi = __reduce_max_sync(kFull, hi);
    if (l == 0) { S.red[w] = lo; S.red[8 + w] = hi; }
    __syncthreads();
    lo = S.red[0]; hi = S.red[8];
#pragma unroll
    for (int u = 1; u < kRowNT / 32; ++u) { lo = min(lo, S.red[u]); hi = max(hi, S.red[8 + u]); }
    *lo_out = lo; *hi_out = hi;
  };
  // the bin of `hist` holding the rem-th largest counted key; rem becomes the
  // rank inside that bin
  auto pick = [&](int& rem) -> uint32_t {
    uint32_t cnt[kRowBPT], tot = 0;
#pragma unroll
    for (int e = 0; e < kRowBPT; e += 4) {
      const uint4 h4 = *reinterpret_cast<const uint4*>(&S.hist[tid * kRowBPT + e]);
      cnt[e] = h4.x; cnt[e + 1] = h4.y; cnt[e + 2] = h4.z; cnt[e + 3] = h4.w;
      tot += h4.x + h4.y + h4.z + h4.w;
    }
    // keys in the bins of the threads after this one: suffix sums within the
    // warp, warp totals through shared memory (one barrier)
    uint32_t suf = tot;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_down_sync(kFull, suf, o);
      if (l + o < 32) suf += y;
    }
    if (l == 0) S.sc[w] = int(suf);
    __syncthreads();
    uint32_t above = suf - tot;
#pragma unroll
    for (int u = 0; u < kRowNT / 32; ++u)
      if (u > w) above += uint32_t(S.sc[u]);
    if (above < uint32_t(rem) && uint32_t(rem) <= above + tot) {
      uint32_t a = uint32_t(above);
#pragma unroll
      for (int e = kRowBPT - 1; e >= 0; --e) {
        if (a + cnt[e] >= uint32_t(rem)) { S.pk[0] = tid * kRowBPT + e; S.pk[1] = int(a); break; }
        a += cnt[e];
      }
    }
    __syncthreads();
    rem -= S.pk[1];
    return uint32_t(S.pk[0]);
  };

  uint32_t ulo, uhi;
  {
    // this thread's key range (keys past nj stand in as the other bound)
    uint32_t lo = 0xffffffffu, hi = 0u;
    if (nj == kRowKPT) {
#pragma unroll
      for (int c = 0; c < kRowChunks; ++c) {
        const uint4 v = chunk(c);
        lo = __vimin3_u32(lo, v.x, __vimin3_u32(v.y, v.z, v.w));
        hi = __vimax3_u32(hi, v.x, __vimax3_u32(v.y, v.z, v.w));
      }
    } else {
#pragma unroll
      for (int c = 0; c < kRowChunks; ++c) {
        const uint4 v = chunk(c);
        const uint32_t a0 = 4 * c < nj ? v.x : 0xffffffffu, a1 = 4 * c + 1 < nj ? v.y : 0xffffffffu;
        const uint32_t a2 = 4 * c + 2 < nj ? v.z : 0xffffffffu, a3 = 4 * c + 3 < nj ? v.w : 0xffffffffu;
        const uint32_t b0 = 4 * c < nj ? v.x : 0u, b1 = 4 * c + 1 < nj ? v.y : 0u;
        const uint32_t b2 = 4 * c + 2 < nj ? v.z : 0u, b3 = 4 * c + 3 < nj ? v.w : 0u;
        lo = __vimin3_u32(lo, a0, __vimin3_u32(a1, a2, a3));
        hi = __vimax3_u32(hi, b0, __vimax3_u32(b1, b2, b3));
      }
    }
    block_min_max(lo, hi, &ulo, &uhi);
  }
  int rem = k;
  uint32_t T = 0;
  int take_eq = 0;
  uint32_t gtm = 0, eqm = 0;  // this thread's keys above T, and equal to T (bit j: key j)
  bool done = false;
  const float flo = key_score(ulo), fhi = key_score(uhi);
  const float c = float(kRowBins - 3) / (fhi - flo);
  if (flo < fhi && c > 0.f && c < INFINITY) {
    // the bin of score x: (x - lo) * c + 1 rounded to an integer by adding
    // 1.5 * 2^23 in one fma and reading the low bits of the sum (the sum stays
    // positive, and positive float bit patterns grow with the value, so the
    // bin never decreases as x grows). When the row's smallest and largest
    // keys land in [0, kRowBins), every key does; otherwise bins are clamped.
    const float nb = 12582913.0f - flo * c;
    uint32_t vbr[kRowKPT / 2];  // the bins of keys 2r and 2r + 1
    const int blo = int(__float_as_uint(fmaf(flo, c, nb)) - 0x4B400000u);
    const int bhi = int(__float_as_uint(fmaf(fhi, c, nb)) - 0x4B400000u);
    if (blo >= 0 && bhi < kRowBins) {
      // the slots past this thread's candidates read as the row's smallest
      // key (so every thread takes the same path), and the smallest key's
      // bin gives those kRowCap - n counts back
      for (int j = nj; j < kRowKPT; ++j)
        reinterpret_cast<uint32_t*>(&S.keys[(tid << 3) | ((j >> 2) ^ (tid & 7))])[j & 3] = ulo;
      if (tid == 0) atomicSub(&S.hist[blo], uint32_t(kRowCap - n));
#pragma unroll
      for (int cc = 0; cc < kRowChunks; ++cc) {
        const uint4 v = chunk(cc);
        const uint32_t b0 = __float_as_uint(fmaf(key_score(v.x), c, nb)) - 0x4B400000u;
        const uint32_t b1 = __float_as_uint(fmaf(key_score(v.y), c, nb)) - 0x4B400000u;
        const uint32_t b2 = __float_as_uint(fmaf(key_score(v.z), c, nb)) - 0x4B400000u;
        const uint32_t b3 = __float_as_uint(fmaf(key_score(v.w), c, nb)) - 0x4B400000u;
        atomicAdd(&S.hist[b0], 1u);
        atomicAdd(&S.hist[b1], 1u);
        atomicAdd(&S.hist[b2], 1u);
        atomicAdd(&S.hist[b3], 1u);
        vbr[2 * cc] = __byte_perm(b0, b1, 0x5410);
        vbr[2 * cc + 1] = __byte_perm(b2, b3, 0x5410);
      }
    } else {
#pragma unroll
      for (int r = 0; r < kRowKPT / 2; ++r) vbr[r] = 0;
      each([&](int j, uint32_t u) {
        const int bi = int(__float_as_uint(fmaf(key_score(u), c, nb)) - 0x4B400000u);
        const uint32_t b = uint32_t(min(kRowBins - 1, max(0, bi)));
        if (j < nj) atomicAdd(&S.hist[b], 1u);
        vbr[j >> 1] |= b << (16 * (j & 1));
      });
    }
    __syncthreads();
    const uint32_t bin = pick(rem);
    const uint32_t cstar = S.hist[bin];
    // keys in bins above the threshold bin, and keys inside it, two per
    // subtraction: with bit 15 of each 11-bit half set, subtracting bin + 1
    // (bin) from both halves leaves bit 15 set exactly where the half's bin is
    // above (at least) the threshold bin; the flags of keys 2r and 2r + 1 are
    // collected in bits r and 16 + r, then interleaved into key order
    const uint32_t above2 = (bin + 1u) * 0x10001u, atleast2 = bin * 0x10001u;
    uint32_t gtp = 0, gep = 0;
#pragma unroll
    for (int r = 0; r < kRowKPT / 2; ++r) {
      const uint32_t x = vbr[r] | 0x80008000u;
      gtp |= ((x - above2) >> (15 - r)) & (0x10001u << r);
      gep |= ((x - atleast2) >> (15 - r)) & (0x10001u << r);
    }
    gtm = interleave_halves(gtp) & jmask;
    uint32_t binm = interleave_halves(gep & ~gtp) & jmask;
    if (cstar <= uint32_t(kRowRank)) {
      // gather the bin and rank it pairwise: T is its rem-th largest key
      for (uint32_t mm = binm; mm; mm &= mm - 1u) S.list[atomicAdd(&S.red[16], 1u)] = key_at(__ffs(mm) - 1);
      __syncthreads();
      if (tid < int(cstar)) {
        const uint32_t x = S.list[tid];
        int gt = 0, ge = 0;
        for (int q = 0; q < int(cstar); ++q) {
          const uint32_t y = S.list[q];
          gt += y > x;
          ge += y >= x;
        }
        if (gt < rem && rem <= ge) { S.red[17] = x; S.red[18] = uint32_t(rem - gt); }  // writers agree
      }
      __syncthreads();
      T = S.red[17];
      take_eq = int(S.red[18]);
      for (uint32_t mm = binm; mm; mm &= mm - 1u) {
        const int j = __ffs(mm) - 1;
        const uint32_t u = key_at(j);
        gtm |= uint32_t(u > T) << j;
        eqm |= uint32_t(u == T) << j;
      }
      done = true;
    } else {
      // a crowded bin: its key range, then rounds on the key bits inside it
      uint32_t lo = 0xffffffffu, hi = 0u;
      for (uint32_t mm = binm; mm; mm &= mm - 1u) {
        const uint32_t u = key_at(__ffs(mm) - 1);
        lo = min(lo, u);
        hi = max(hi, u);
      }
      __syncthreads();  // every thread has read hist[bin] before red[] and hist are reused
      block_min_max(lo, hi, &ulo, &uhi);
    }
  }
  if (!done) {
    // 11-bit rounds over the key range [ulo, uhi] that holds the threshold
    uint32_t base = ulo, width = uhi - ulo;
    for (;;) {
      const int bits = 32 - __clz(width);
      const int shift = bits > 11 ? bits - 11 : 0;
      for (int e = 0; e < kRowBPT; ++e) S.hist[tid * kRowBPT + e] = 0;
      __syncthreads();
      each([&](int j, uint32_t u) {
        const uint32_t d = u - base;
        if (j < nj && d <= width) atomicAdd(&S.hist[d >> shift], 1u);
      });
      __syncthreads();
      const uint32_t bin = pick(rem);
      const bool whole = S.hist[bin] == uint32_t(rem);
      base += bin << shift;
      width = min(shift ? (1u << shift) - 1u : 0u, uhi - base);
      __syncthreads();
      if (whole && base > 0u) { T = base - 1u; take_eq = 0; break; }
      if (shift == 0) { T = base; take_eq = rem; break; }
    }
    gtm = eqm = 0;
    each([&](int j, uint32_t u) {
      if (j < nj) {
        gtm |= uint32_t(u > T) << j;
        eqm |= uint32_t(u == T) << j;
      }
    });
  }
  // emit in position order: slot = (#keys > T before) + min(#keys == T before, take_eq)
  // keys before this thread's: prefix sums within the warp, warp totals
  // through shared memory (one barrier); both counts < 2^14
  const int mine = (__popc(gtm) << 16) | __popc(eqm);
  int incl = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(kFull, incl, o);
    if (l >= o) incl += y;
  }
  if (l == 31) S.sc[8 + w] = incl;
  __syncthreads();
  int before = incl - mine;
#pragma unroll
  for (int u = 0; u < kRowNT / 32; ++u)
    if (u < w) before += S.sc[8 + u];
  const int G = before >> 16, Q = before & 0xffff;
  // the keys equal to T that are taken: the first take_eq - Q of this thread's
  uint32_t sel = gtm;
  for (uint32_t mm = eqm, q = uint32_t(Q); mm && q < uint32_t(take_eq); mm &= mm - 1u, ++q) sel |= mm & (0u - mm);
  // The row's k indices are assembled in shared memory (over the keys, which
  // every thread has finished reading: the barrier above) and then written
  // out with coalesced stores. This thread's 32 positions lie in one kept
  // block when B >= 32; its selected tokens are then tok0 + j, in
  // consecutive slots.
  int32_t* so = reinterpret_cast<int32_t*>(S.keys);
  int32_t* o = so + G + min(Q, take_eq);
  if (B >= kRowKPT) {
    const int32_t tok0 = (S.blk[p0 >> lb] << lb) + (p0 & (B - 1));
    for (uint32_t mm = sel; mm; mm &= mm - 1u) *o++ = tok0 + (__ffs(mm) - 1);
  } else {
    for (uint32_t mm = sel; mm; mm &= mm - 1u) {
      const int p = p0 + __ffs(mm) - 1;
      *o++ = (S.blk[p >> lb] << lb) + (p & (B - 1));
    }
  }
  __syncthreads();
  if ((k & 3) == 0 && (reinterpret_cast<uintptr_t>(out) & 15u) == 0) {
    for (int e = tid; e < k / 4; e += kRowNT)
      reinterpret_cast<int4*>(out)[e] = reinterpret_cast<const int4*>(so)[e];
  } else {
    for (int e = tid; e < k; e += kRowNT) out[e] = so[e];
  }
}

}  // namespace

// Keys per thread for up to n keys over NT threads: 1, 2, 4, ..., 64.
static int keys_per_thread(int64_t n) {
  int kpt = 1;
  while (int64_t(kpt) * NT < n) kpt *= 2;
  return kpt;
}

#define HSA_KPT_DISPATCH(kpt, CALL) \
  switch (kpt) {                    \
    case 1: CALL(1); break;         \
    case 2: CALL(2); break;         \
    case 4: CALL(4); break;         \
    case 8: CALL(8); break;         \
    case 16: CALL(16); break;       \
    case 32: CALL(32); break;       \
    default: CALL(64); break;       \
  }

void launch_topm_from_keys(RowMap rm, int64_t rows, const uint32_t* bkeys, int64_t ld, int B, int m,
                           int64_t max_cand, int32_t* blocks, cudaStream_t s, bool pdl) {
  if (rows == 0) return;
  count_launches(1);
  if (max_cand <= 512 && rows >= 8 * int64_t(num_sms())) {
    // many rows of few candidates: one warp per row
    const unsigned grid = unsigned((rows + kTopmWarpsPerCta - 1) / kTopmWarpsPerCta);
    if (max_cand <= 256)
      launch_kernel(pdl, topm_warp_rows_kernel<8>, grid, 32 * kTopmWarpsPerCta, 0, s, rm, rows, bkeys, ld, B, m,
                    blocks);
    else
      launch_kernel(pdl, topm_warp_rows_kernel<16>, grid, 32 * kTopmWarpsPerCta, 0, s, rm, rows, bkeys, ld, B, m,
                    blocks);
    return;
  }
#define HSA_TOPM(K) launch_kernel(pdl, topm_from_keys_kernel<K>, unsigned(rows), NT, 0, s, rm, bkeys, ld, B, m, blocks)
  HSA_KPT_DISPATCH(keys_per_thread(max_cand), HSA_TOPM)
#undef HSA_TOPM
}

void launch_pair_lists(RowMap rm, int64_t rows, const int32_t* blocks, int B, int m, int k, int nbins,
                       int* cnt, int* off, int* cursor, int4* tiles, int* ntiles, uint32_t* pairs,
                       cudaStream_t s) {
  if (rows == 0) return;
  count_launches(3);
  cudaMemsetAsync(cnt, 0, sizeof(int) * nbins, s);
  int rpc = kPairRows;
  while (rpc > 16 && (rows + rpc - 1) / rpc < 2 * int64_t(num_sms())) rpc /= 2;
  const unsigned grid = unsigned((rows + rpc - 1) / rpc);
  const size_t smem1 = sizeof(int) * nbins, smem2 = 2 * sizeof(int) * nbins;
  cudaFuncSetAttribute(pair_bin_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem1));
  cudaFuncSetAttribute(pair_bin_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem2));
  pair_bin_kernel<false><<<grid, NT, smem1, s>>>(rm, rows, blocks, B, m, k, nbins, rpc, cnt, nullptr, nullptr,
                                                 nullptr, nullptr);
  // the scan and the scatter pass overlap their launches with their predecessors
  launch_kernel(true, pair_scan_kernel, 1, 1024, 0, s, nbins, cnt, off, cursor, ntiles);
  launch_kernel(true, pair_bin_kernel<true>, grid, NT, smem2, s, rm, rows, blocks, B, m, k, nbins, rpc, cnt,
                static_cast<const int*>(off), cursor, pairs, tiles);
}

void launch_topk_from_keys(RowMap rm, int64_t rows, const int32_t* blocks, const uint32_t* tkeys, int B,
                           int m, int k, int32_t* indices, cudaStream_t s, bool pdl) {
  if (rows == 0) return;
  count_launches(1);
  if (int64_t(m) * B <= kRowCap && (B & (B - 1)) == 0 && B >= 4 && m <= 256 &&
      (reinterpret_cast<uintptr_t>(tkeys) & 15u) == 0) {
    // rows of up to 8192 candidates: a 256-thread CTA per row, the row staged in shared memory
    cudaFuncSetAttribute(topk_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(sizeof(RowSmem)));
    launch_kernel(pdl, topk_rows_kernel, unsigned(rows), kRowNT, sizeof(RowSmem), s, rm, blocks, tkeys, B, m, k,
                  indices);
  } else if (rows < 2 * num_sms()) {
    // few longer rows (a decode batch): wide CTAs cut each row's latency
#define HSA_TOPK(K) \
  launch_kernel(pdl, topk_from_keys_kernel<1024, K>, unsigned(rows), 1024, 0, s, rm, blocks, tkeys, B, m, k, indices)
    int kpt = 1;
    while (int64_t(kpt) * 1024 < int64_t(m) * B) kpt *= 2;
    HSA_KPT_DISPATCH(kpt, HSA_TOPK)
#undef HSA_TOPK
  } else {
    // many longer rows: one warp per row
    const int smem = kWarpRowsPerCta * (kWBins + kMaxRowBlocks) * 4;
    cudaFuncSetAttribute(topk_warp_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    topk_warp_rows_kernel<<<unsigned((rows + kWarpRowsPerCta - 1) / kWarpRowsPerCta), 32 * kWarpRowsPerCta, smem,
                            s>>>(rm, rows, blocks, tkeys, B, m, k, indices);
  }
}

}  // namespace hsa
