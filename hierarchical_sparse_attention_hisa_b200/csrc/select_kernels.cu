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

namespace hsa {
namespace {

constexpr int NT = 256;
constexpr int NT_TOPK = 512;  // top-k rows hold up to m*B keys: 16 per thread at 8192

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

template <int KPT>
__global__ void __launch_bounds__(NT) topm_from_keys_kernel(RowMap rm, const uint32_t* __restrict__ bkeys,
                                                           int64_t ld, int B, int m, int32_t* __restrict__ blocks) {
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
  load_keys<KPT>(bkeys + i * ld + 1, n, key);
  RegSelect<NT, KPT> rs{hist, scratch};
  uint32_t T;
  int take_eq;
  rs.threshold(key, n, m - 2, &T, &take_eq);
  if (threadIdx.x == 0) { out[0] = 0; out[m - 1] = int32_t(nb - 1); }
  rs.compact(key, n, T, take_eq, [&](int rank, int c) { out[1 + rank] = c + 1; });
}

// Pairs of the rows [r0, r0 + ROWS) that need token scores, binned by block.
constexpr int kPairRows = 64;

template <bool SCATTER>
__global__ void __launch_bounds__(NT) pair_bin_kernel(RowMap rm, int64_t rows, const int32_t* __restrict__ blocks,
                                                     int B, int m, int k, int nbins, int* __restrict__ cnt,
                                                     const int* __restrict__ off, int* __restrict__ cursor,
                                                     uint32_t* __restrict__ pairs) {
  extern __shared__ int sh[];
  int* hist = sh;             // [nbins]
  int* base = sh + nbins;     // [nbins] (scatter only)
  for (int b = threadIdx.x; b < nbins; b += NT) hist[b] = 0;
  __syncthreads();
  const int64_t r0 = int64_t(blockIdx.x) * kPairRows;
  // one warp per row at a time; lanes over slots
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto row_pairs = [&](auto&& fn) {
    for (int rr = warp; rr < kPairRows; rr += NT / 32) {
      const int64_t i = r0 + rr;
      if (i >= rows) break;
      const int32_t* blk = blocks + i * m;
      const int64_t t = rm.pos(i);
      int nblk = 0, ncand = 0;
      if (!row_candidates(blk, m, t, B, &nblk, &ncand) || ncand <= k) continue;
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
  __syncthreads();
  row_pairs([&](int64_t i, int s, int b) {
    const int pos = base[b] + atomicAdd(&hist[b], 1);
    pairs[pos] = uint32_t(i) * uint32_t(m) + uint32_t(s);
  });
}

// Single CTA: offsets of every bin, the tile table (block, first pair,
// pair count) in tiles of <= 128 pairs, and the tile count.
__global__ void __launch_bounds__(1024) pair_scan_kernel(int nbins, const int* __restrict__ cnt, int* __restrict__ off,
                                                        int* __restrict__ cursor, int4* __restrict__ tiles,
                                                        int* __restrict__ ntiles) {
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
      const int o = carry_pairs + ep;
      off[b] = o;
      cursor[b] = 0;
      for (int u = 0; u < nt; ++u)
        tiles[carry_tiles + et + u] = make_int4(b, o + 128 * u, min(128, c - 128 * u), 0);
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
  __shared__ uint32_t hist[RegSelect<NT, KPT>::kBins];
  __shared__ int scratch[NT / 32 + 8];
  __shared__ int blk[256];
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
                           int64_t max_cand, int32_t* blocks, cudaStream_t s) {
  if (rows == 0) return;
  count_launches(1);
#define HSA_TOPM(K) topm_from_keys_kernel<K><<<unsigned(rows), NT, 0, s>>>(rm, bkeys, ld, B, m, blocks)
  HSA_KPT_DISPATCH(keys_per_thread(max_cand), HSA_TOPM)
#undef HSA_TOPM
}

void launch_pair_lists(RowMap rm, int64_t rows, const int32_t* blocks, int B, int m, int k, int nbins,
                       int* cnt, int* off, int* cursor, int4* tiles, int* ntiles, uint32_t* pairs,
                       cudaStream_t s) {
  if (rows == 0) return;
  count_launches(3);
  cudaMemsetAsync(cnt, 0, sizeof(int) * nbins, s);
  const unsigned grid = unsigned((rows + kPairRows - 1) / kPairRows);
  const size_t smem1 = sizeof(int) * nbins, smem2 = 2 * sizeof(int) * nbins;
  cudaFuncSetAttribute(pair_bin_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem1));
  cudaFuncSetAttribute(pair_bin_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem2));
  pair_bin_kernel<false><<<grid, NT, smem1, s>>>(rm, rows, blocks, B, m, k, nbins, cnt, nullptr, nullptr, nullptr);
  pair_scan_kernel<<<1, 1024, 0, s>>>(nbins, cnt, off, cursor, tiles, ntiles);
  pair_bin_kernel<true><<<grid, NT, smem2, s>>>(rm, rows, blocks, B, m, k, nbins, cnt, off, cursor, pairs);
}

void launch_topk_from_keys(RowMap rm, int64_t rows, const int32_t* blocks, const uint32_t* tkeys, int B,
                           int m, int k, int32_t* indices, cudaStream_t s) {
  if (rows == 0) return;
  count_launches(1);
  // few rows (a decode batch): wide CTAs cut each row's latency; many rows:
  // 512 threads keep several CTAs per SM
  if (rows < 2 * num_sms()) {
#define HSA_TOPK(K) topk_from_keys_kernel<1024, K><<<unsigned(rows), 1024, 0, s>>>(rm, blocks, tkeys, B, m, k, indices)
    int kpt = 1;
    while (int64_t(kpt) * 1024 < int64_t(m) * B) kpt *= 2;
    HSA_KPT_DISPATCH(kpt, HSA_TOPK)
#undef HSA_TOPK
  } else {
#define HSA_TOPK(K) topk_from_keys_kernel<NT_TOPK, K><<<unsigned(rows), NT_TOPK, 0, s>>>(rm, blocks, tkeys, B, m, k, indices)
    int kpt = 1;
    while (int64_t(kpt) * NT_TOPK < int64_t(m) * B) kpt *= 2;
    HSA_KPT_DISPATCH(kpt, HSA_TOPK)
#undef HSA_TOPK
  }
}

}  // namespace hsa
