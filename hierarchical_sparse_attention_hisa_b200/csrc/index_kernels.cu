// HISA indexer kernels: block representatives, block-level selection and
// token-level selection (page "HISA: Hierarchical Indexed Sparse Attention",
// sections 第一步 and 第二步, forced first/last block note).
#include "kernels.cuh"

namespace hsa {

// ---------------------------------------------------------------------------
// Block sums: ksum[b][c] = sum_{j = bB}^{bB+B-1} k_idx[j][c] in fp32.
// One CTA per complete block; 128-bit loads of 8 bf16 columns; the CTA's
// row lanes each sum a strided subset of the block's rows and are reduced
// in shared memory. Integer-valued inputs give exact sums in any order.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) block_sums_kernel(const uint4* __restrict__ k_idx, int B,
                                                         int64_t nbc, float* __restrict__ ksum) {
  constexpr int CG = D / 8;        // 16-byte column groups per row
  constexpr int RL = 256 / CG;     // row lanes
  __shared__ float red[RL][D + 1];
  const int64_t b = blockIdx.x;
  if (b >= nbc) return;
  const int cg = threadIdx.x % CG, rl = threadIdx.x / CG;
  float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  for (int r = rl; r < B; r += RL) {
    const uint4 v = __ldg(k_idx + (b * B + r) * CG + cg);
    acc[0] += bf16_lo(v.x); acc[1] += bf16_hi(v.x);
    acc[2] += bf16_lo(v.y); acc[3] += bf16_hi(v.y);
    acc[4] += bf16_lo(v.z); acc[5] += bf16_hi(v.z);
    acc[6] += bf16_lo(v.w); acc[7] += bf16_hi(v.w);
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) red[rl][cg * 8 + e] = acc[e];
  __syncthreads();
  for (int c = threadIdx.x; c < D; c += 256) {
    float s = 0.f;
    for (int l = 0; l < RL; ++l) s += red[l][c];
    ksum[b * D + c] = s;
  }
}

void launch_block_sums(const void* k_idx, int64_t Lk, int B, int d_idx, float* ksum,
                       cudaStream_t s) {
  const int64_t nbc = Lk / B;
  if (nbc == 0) return;
  count_launches(1);
  if (d_idx == 128)
    block_sums_kernel<128><<<unsigned(nbc), 256, 0, s>>>((const uint4*)k_idx, B, nbc, ksum);
  else
    block_sums_kernel<64><<<unsigned(nbc), 256, 0, s>>>((const uint4*)k_idx, B, nbc, ksum);
}

// ---------------------------------------------------------------------------
// Three bf16 planes hi + mid + lo whose sum is the fp32 block sum (the
// tensor-core block scoring multiplies each plane by bf16 queries; the
// products are exact and the three partial dot products add up in fp32).
// ---------------------------------------------------------------------------
__global__ void ksum_split_kernel(const float* __restrict__ ksum, int64_t n, uint16_t* __restrict__ split) {
  griddep_wait();
  griddep_launch();
  for (int64_t e = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; e < n; e += int64_t(gridDim.x) * blockDim.x) {
    const float x = ksum[e];
    const uint32_t hi = f32_to_bf16_rn(x);
    const float r1 = x - __uint_as_float(hi << 16);
    const uint32_t mid = f32_to_bf16_rn(r1);
    const float r2 = r1 - __uint_as_float(mid << 16);
    split[e] = uint16_t(hi);
    split[n + e] = uint16_t(mid);
    split[2 * n + e] = uint16_t(f32_to_bf16_rn(r2));
  }
}

void launch_ksum_split(const float* ksum, int64_t n, void* split, cudaStream_t s) {
  if (n == 0) return;
  count_launches(1);
  const int64_t blocks = (n + 255) / 256;
  launch_kernel(true, ksum_split_kernel, unsigned(blocks < 4096 ? blocks : 4096), 256, 0, s, ksum, n,
                (uint16_t*)split);
}

// ---------------------------------------------------------------------------
// Block selection, one CTA per query row. Candidate c is block c+1 of
// 1 .. nb-2; its score q . ksum[c+1] is an fp32 dot product (q widened
// exactly from bf16). The m-2 best candidates by (score desc, block asc) are
// kept with the forced blocks 0 and nb-1, ascending.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) select_blocks_kernel(RowMap rm, const uint16_t* __restrict__ q_idx,
                                                            const float* __restrict__ ksum,
                                                            int64_t ksum_seq_stride, int B, int m,
                                                            int32_t* __restrict__ blocks) {
  constexpr int NT = 256;
  extern __shared__ __align__(16) uint32_t smem_u32[];
  __shared__ uint32_t hist[RadixSelect<NT>::kBins];
  __shared__ int scratch[NT / 32 + 8];
  __shared__ float qs[D];
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
  if (m == 2) {  // only the two forced blocks are kept
    if (threadIdx.x == 0) { out[0] = 0; out[1] = int32_t(nb - 1); }
    return;
  }
  for (int c = threadIdx.x; c < D; c += NT) qs[c] = __uint_as_float(uint32_t(q_idx[i * D + c]) << 16);
  __syncthreads();
  const float* ks = ksum + (rm.ctx ? i * ksum_seq_stride : 0);
  const int n = int(nb - 2);
  uint32_t* keys = smem_u32;
  for (int c = threadIdx.x; c < n; c += NT) {
    const float4* row = reinterpret_cast<const float4*>(ks + int64_t(c + 1) * D);
    float acc = 0.f;
#pragma unroll 4
    for (int e = 0; e < D / 4; ++e) {
      const float4 v = __ldg(row + e);
      acc = __fmaf_rn(qs[4 * e + 0], v.x, acc);
      acc = __fmaf_rn(qs[4 * e + 1], v.y, acc);
      acc = __fmaf_rn(qs[4 * e + 2], v.z, acc);
      acc = __fmaf_rn(qs[4 * e + 3], v.w, acc);
    }
    keys[c] = score_key(acc);
  }
  __syncthreads();
  RadixSelect<NT> rs{hist, scratch};
  uint32_t T;
  int take_eq;
  rs.threshold(keys, n, m - 2, &T, &take_eq);
  if (threadIdx.x == 0) { out[0] = 0; out[m - 1] = int32_t(nb - 1); }
  rs.compact(keys, n, T, take_eq, [&](int rank, int c) { out[1 + rank] = c + 1; });
}

void launch_select_blocks(RowMap rm, int64_t rows, const void* q_idx, const float* ksum,
                          int64_t ksum_seq_stride, int B, int m, int d_idx, int32_t* blocks,
                          int64_t max_cand, cudaStream_t s) {
  if (rows == 0) return;
  count_launches(1);
  const size_t smem = size_t(max_cand > 0 ? max_cand : 1) * 4;
  if (d_idx == 128) {
    cudaFuncSetAttribute(select_blocks_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    select_blocks_kernel<128><<<unsigned(rows), 256, smem, s>>>(rm, (const uint16_t*)q_idx, ksum,
                                                                ksum_seq_stride, B, m, blocks);
  } else {
    cudaFuncSetAttribute(select_blocks_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    select_blocks_kernel<64><<<unsigned(rows), 256, smem, s>>>(rm, (const uint16_t*)q_idx, ksum,
                                                               ksum_seq_stride, B, m, blocks);
  }
}

// ---------------------------------------------------------------------------
// Token selection, one CTA per query row. Candidates are enumerated in block
// order (blocks ascending, the own block last), so candidate c is token
// blocks[c / B] * B + c % B and candidates are ascending in j; the own
// block is cut at j <= t. Scores q . k_idx[j] are fp32 dot products of
// exactly widened bf16 values; the k best by (score desc, j asc) are
// written ascending.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) select_tokens_kernel(RowMap rm, const uint16_t* __restrict__ q_idx,
                                                            const uint16_t* __restrict__ k_idx,
                                                            const int32_t* __restrict__ blocks, int B,
                                                            int m, int k, int32_t* __restrict__ indices) {
  constexpr int NT = 256;
  extern __shared__ __align__(16) uint32_t smem_u32[];
  __shared__ uint32_t hist[RadixSelect<NT>::kBins];
  __shared__ int scratch[NT / 32 + 8];
  __shared__ float qs[D];
  __shared__ int blk[512];
  __shared__ int s_nblk;
  const int64_t i = blockIdx.x;
  int32_t* out = indices + i * int64_t(k);
  if (!rm.valid(i)) {
    for (int s = threadIdx.x; s < k; s += NT) out[s] = -1;
    return;
  }
  const int64_t t = rm.pos(i);
  const uint16_t* kbase = k_idx + rm.seq_row0(i) * D;
  if (threadIdx.x == 0) s_nblk = 0;
  __syncthreads();
  for (int s = threadIdx.x; s < m; s += NT) {
    const int b = blocks[i * m + s];
    blk[s] = b;
    if (b >= 0) atomicAdd(&s_nblk, 1);
  }
  for (int c = threadIdx.x; c < D; c += NT) qs[c] = __uint_as_float(uint32_t(q_idx[i * D + c]) << 16);
  __syncthreads();
  const int nblk = s_nblk;
  // The block list must be the selector's: ascending, valid ids first, the
  // query's own block last. Anything else yields an all -1 row (no reads).
  bool ok = nblk > 0 && blk[nblk - 1] == int(t / B);
  for (int s = 0; s + 1 < nblk && ok; ++s) ok = blk[s] >= 0 && blk[s] < blk[s + 1];
  if (!ok) {
    for (int s = threadIdx.x; s < k; s += NT) out[s] = -1;
    return;
  }
  const int64_t own = blk[nblk - 1];
  const int n = int((nblk - 1) * int64_t(B) + (t - own * B + 1));
  auto tok = [&](int c) -> int64_t { return int64_t(blk[c / B]) * B + c % B; };
  if (n <= k) {
    for (int s = threadIdx.x; s < k; s += NT) out[s] = s < n ? int32_t(tok(s)) : -1;
    return;
  }
  uint32_t* keys = smem_u32;
  for (int c = threadIdx.x; c < n; c += NT) {
    const uint4* row = reinterpret_cast<const uint4*>(kbase + tok(c) * D);
    float acc = 0.f;
#pragma unroll 4
    for (int e = 0; e < D / 8; ++e) {
      const uint4 v = __ldg(row + e);
      acc = __fmaf_rn(qs[8 * e + 0], bf16_lo(v.x), acc);
      acc = __fmaf_rn(qs[8 * e + 1], bf16_hi(v.x), acc);
      acc = __fmaf_rn(qs[8 * e + 2], bf16_lo(v.y), acc);
      acc = __fmaf_rn(qs[8 * e + 3], bf16_hi(v.y), acc);
      acc = __fmaf_rn(qs[8 * e + 4], bf16_lo(v.z), acc);
      acc = __fmaf_rn(qs[8 * e + 5], bf16_hi(v.z), acc);
      acc = __fmaf_rn(qs[8 * e + 6], bf16_lo(v.w), acc);
      acc = __fmaf_rn(qs[8 * e + 7], bf16_hi(v.w), acc);
    }
    keys[c] = score_key(acc);
  }
  __syncthreads();
  RadixSelect<NT> rs{hist, scratch};
  uint32_t T;
  int take_eq;
  rs.threshold(keys, n, k, &T, &take_eq);
  rs.compact(keys, n, T, take_eq, [&](int rank, int c) { out[rank] = int32_t(tok(c)); });
}

void launch_select_tokens(RowMap rm, int64_t rows, const void* q_idx, const void* k_idx,
                          const int32_t* blocks, int B, int m, int k, int d_idx, int32_t* indices,
                          int64_t max_cand, cudaStream_t s) {
  if (rows == 0) return;
  count_launches(1);
  const size_t smem = size_t(max_cand) * 4;
  if (d_idx == 128) {
    cudaFuncSetAttribute(select_tokens_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    select_tokens_kernel<128><<<unsigned(rows), 256, smem, s>>>(
        rm, (const uint16_t*)q_idx, (const uint16_t*)k_idx, blocks, B, m, k, indices);
  } else {
    cudaFuncSetAttribute(select_tokens_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    select_tokens_kernel<64><<<unsigned(rows), 256, smem, s>>>(
        rm, (const uint16_t*)q_idx, (const uint16_t*)k_idx, blocks, B, m, k, indices);
  }
}

}  // namespace hsa
