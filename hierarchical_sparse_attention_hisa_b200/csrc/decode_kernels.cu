// Decode-step kernels: block scores of each sequence's new query (whose first
// CTA also appends the new token to the caller's caches and writes the block
// sum of a block the token completes), token scores inside the kept blocks,
// and the combination of a split attention's parts (which also advances the
// per-sequence lengths once every earlier kernel of the step has read them).
#include <algorithm>

#include "kernels.cuh"

namespace hsa {

// The caches the append writes and the new token's rows.
struct AppendArgs {
  uint16_t *k_idx_cache, *K_cache, *V_cache;
  float* ksum_cache;
  const uint16_t *k_idx_new, *K_new, *V_new;
  int DA;
};

// Appends sequence b's new token at position t (all threads of the CTA take
// part) and writes the block sum of a block the token completes.
template <int DI>
__device__ void append_token(const AppendArgs& a, int64_t b, int64_t t, int64_t capacity, int B) {
  const int tid = threadIdx.x, nt = blockDim.x;
  const int64_t row = b * capacity + t;
  for (int e = tid; e < DI / 8; e += nt)
    reinterpret_cast<uint4*>(a.k_idx_cache + row * DI)[e] = reinterpret_cast<const uint4*>(a.k_idx_new + b * DI)[e];
  for (int e = tid; e < a.DA / 8; e += nt) {
    reinterpret_cast<uint4*>(a.K_cache + row * a.DA)[e] = reinterpret_cast<const uint4*>(a.K_new + b * a.DA)[e];
    reinterpret_cast<uint4*>(a.V_cache + row * a.DA)[e] = reinterpret_cast<const uint4*>(a.V_new + b * a.DA)[e];
  }
  if ((t + 1) % B != 0) return;
  const int64_t blk = t / B;
  for (int c = tid; c < DI; c += nt) {
    float s = 0.f;
    for (int64_t j = blk * B; j < t; ++j)
      s += __uint_as_float(uint32_t(a.k_idx_cache[(b * capacity + j) * DI + c]) << 16);
    s += __uint_as_float(uint32_t(a.k_idx_new[b * DI + c]) << 16);
    a.ksum_cache[(b * (capacity / B) + blk) * DI + c] = s;
  }
}

// Block scores of the new query of sequence b against its complete blocks
// 1 .. nb-2 (blocks 0 and nb-1 are forced, so never scored): one warp per
// block row of the fp32 block-sum cache, fp32 products reduced across the
// warp, written as order-preserving keys bkeys[b][block].
template <int DI>
__global__ void __launch_bounds__(256) decode_block_scores_kernel(const int32_t* __restrict__ ctx, int64_t capacity,
                                                                  int B, int m, int per_cta,
                                                                  const uint16_t* __restrict__ q_new,
                                                                  const float* __restrict__ ksum_cache,
                                                                  uint32_t* __restrict__ bkeys, int64_t ld,
                                                                  AppendArgs ap) {
  griddep_wait();
  griddep_launch();
  constexpr int VPL = DI / 32;  // fp32 values per lane
  const int64_t b = blockIdx.x;
  const int64_t t = ctx[b];
  if (t < 0 || t >= capacity) return;
  // the first CTA of each sequence appends the new token; the block sum it may
  // write is the own block's, which the scores below never read
  if (blockIdx.y == 0) append_token<DI>(ap, b, t, capacity, B);
  const int64_t nb = t / B + 1;
  if (nb <= m) return;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float q[VPL];
#pragma unroll
  for (int e = 0; e < VPL; ++e) q[e] = __uint_as_float(uint32_t(q_new[b * DI + lane * VPL + e]) << 16);
  const int64_t lo = 1 + int64_t(blockIdx.y) * per_cta, hi = min(nb - 1, lo + per_cta);
  const float* base = ksum_cache + b * (capacity / B) * DI;
  // eight block rows per warp in flight before any of them is reduced
  constexpr int U = 8;
  for (int64_t blk0 = lo + warp; blk0 < hi; blk0 += 8 * U) {
    float v[U][VPL];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t blk = blk0 + 8 * u;
      const float* row = base + blk * DI + lane * VPL;
      if constexpr (VPL == 4) {
        const float4 x = blk < hi ? __ldg(reinterpret_cast<const float4*>(row)) : make_float4(0.f, 0.f, 0.f, 0.f);
        v[u][0] = x.x; v[u][1] = x.y; v[u][2] = x.z; v[u][3] = x.w;
      } else {
        const float2 x = blk < hi ? __ldg(reinterpret_cast<const float2*>(row)) : make_float2(0.f, 0.f);
        v[u][0] = x.x; v[u][1] = x.y;
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t blk = blk0 + 8 * u;
      float acc = q[0] * v[u][0];
#pragma unroll
      for (int e = 1; e < VPL; ++e) acc = __fmaf_rn(q[e], v[u][e], acc);
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) acc += __shfl_xor_sync(kFull, acc, o);
      if (lane == 0 && blk < hi) bkeys[b * ld + blk] = score_key(acc);
    }
  }
}

// Token scores of sequence b's new query against the B keys of its kept
// block in slot s: a half-warp per key row (16-byte loads), written as keys
// tkeys[b][s][r]. Rows past the query's position are scored too but never
// read: the selection takes only the first candidate-count entries.
template <int DI>
__global__ void __launch_bounds__(128) decode_token_scores_kernel(const int32_t* __restrict__ ctx, int64_t capacity,
                                                                  int B, int m, const int32_t* __restrict__ blocks,
                                                                  const uint16_t* __restrict__ q_new,
                                                                  const uint16_t* __restrict__ k_idx_cache,
                                                                  uint32_t* __restrict__ tkeys) {
  griddep_wait();
  griddep_launch();
  constexpr int LPR = DI / 8;          // lanes per row (8 bf16 each)
  constexpr int RPW = 32 / LPR;        // rows per warp instruction
  const int64_t b = blockIdx.x;
  const int s = blockIdx.y;
  const int64_t t = ctx[b];
  if (t < 0 || t >= capacity) return;
  const int blk = blocks[b * m + s];
  if (blk < 0) return;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int sub = lane % LPR, rsub = lane / LPR;
  const uint4 qv = __ldg(reinterpret_cast<const uint4*>(q_new + b * DI) + sub);
  const uint32_t qw[4] = {qv.x, qv.y, qv.z, qv.w};
  const uint16_t* kb = k_idx_cache + (b * capacity + int64_t(blk) * B) * DI;
  uint32_t* out = tkeys + (b * m + s) * int64_t(B);
  // eight rows per lane group in flight before any of them is reduced
  constexpr int U = 8;
  for (int r0 = warp * RPW; r0 < B; r0 += 4 * RPW * U) {
    uint4 kv[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int r = r0 + u * 4 * RPW + rsub;
      kv[u] = r < B ? __ldg(reinterpret_cast<const uint4*>(kb + int64_t(r) * DI) + sub) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int r = r0 + u * 4 * RPW + rsub;
      const uint32_t kw[4] = {kv[u].x, kv[u].y, kv[u].z, kv[u].w};
      float acc = 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        acc = __fmaf_rn(bf16_lo(qw[e]), bf16_lo(kw[e]), acc);
        acc = __fmaf_rn(bf16_hi(qw[e]), bf16_hi(kw[e]), acc);
      }
#pragma unroll
      for (int o = LPR / 2; o >= 1; o >>= 1) acc += __shfl_xor_sync(kFull, acc, o);
      if (sub == 0 && r < B) out[r] = score_key(acc);
    }
  }
}

// O[b][h][:] from the parts of a split query: with M the largest part
// maximum, O = sum_p 2^(m_p - M) O_p / sum_p 2^(m_p - M) l_p (log2 units).
// One CTA per (sequence, head), one thread per output element.
__global__ void decode_combine_kernel(int32_t* __restrict__ ctx, int64_t capacity, int H, int D, int parts,
                                      const float* __restrict__ Opart, const float* __restrict__ mpart,
                                      const float* __restrict__ lpart, uint16_t* __restrict__ O) {
  griddep_wait();
  griddep_launch();
  const int64_t b = blockIdx.x / H;
  const int h = blockIdx.x % H;
  // every load issued before any is used: the sequence length, each part's
  // maximum, row sum and output element
  constexpr int PMAX = 16;
  float lv[PMAX], mv[PMAX], ov[PMAX];
#pragma unroll
  for (int p = 0; p < PMAX; ++p) {
    if (p < parts) {
      const int64_t w = b * parts + p;
      lv[p] = lpart[w * H + h];
      mv[p] = mpart[w * H + h];
      ov[p] = Opart[(w * H + h) * D + threadIdx.x];
    }
  }
  // a sequence that took no step has only empty parts (row sums 0): O = 0
  float out = 0.f;
  {
    float M = -INFINITY;
#pragma unroll
    for (int p = 0; p < PMAX; ++p)
      if (p < parts && lv[p] > 0.f) M = fmaxf(M, mv[p]);
    float num = 0.f, den = 0.f;
#pragma unroll
    for (int p = 0; p < PMAX; ++p) {
      if (p < parts && lv[p] > 0.f) {
        const float f = exp2f(mv[p] - M);
        num = __fmaf_rn(f, ov[p], num);
        den = __fmaf_rn(f, lv[p], den);
      }
    }
    out = den > 0.f ? num / den : 0.f;
  }
  O[(b * H + h) * D + threadIdx.x] = uint16_t(f32_to_bf16_rn(out));
  // every earlier kernel of the step has finished reading the lengths: the
  // sequence grows by one token
  if (h == 0 && threadIdx.x == 0) {
    const int32_t t = ctx[b];
    if (t >= 0 && t < capacity) ctx[b] = t + 1;
  }
}

void launch_decode_block_scores(int batch, int64_t capacity, const int32_t* ctx, int B, int m, int d_idx,
                                const void* q_new, const float* ksum_cache, uint32_t* bkeys, int64_t ld,
                                int d, void* k_idx_cache, void* K_cache, void* V_cache, float* ksum_w,
                                const void* k_idx_new, const void* K_new, const void* V_new, cudaStream_t s) {
  if (batch == 0) return;
  const int64_t nbmax = capacity / B;
  const int per_cta = 64;
  const dim3 grid((unsigned)batch, (unsigned)std::max<int64_t>(1, (nbmax + per_cta - 1) / per_cta));
  AppendArgs ap{(uint16_t*)k_idx_cache, (uint16_t*)K_cache, (uint16_t*)V_cache, ksum_w,
                (const uint16_t*)k_idx_new, (const uint16_t*)K_new, (const uint16_t*)V_new, d};
  count_launches(1);
  if (d_idx == 128)
    launch_kernel(true, decode_block_scores_kernel<128>, grid, 256, 0, s, ctx, capacity, B, m, per_cta,
                  (const uint16_t*)q_new, (const float*)ksum_cache, bkeys, ld, ap);
  else
    launch_kernel(true, decode_block_scores_kernel<64>, grid, 256, 0, s, ctx, capacity, B, m, per_cta,
                  (const uint16_t*)q_new, (const float*)ksum_cache, bkeys, ld, ap);
}

void launch_decode_token_scores(int batch, int64_t capacity, const int32_t* ctx, int B, int m, int d_idx,
                                const int32_t* blocks, const void* q_new, const void* k_idx_cache,
                                uint32_t* tkeys, cudaStream_t s) {
  if (batch == 0) return;
  const dim3 grid((unsigned)batch, (unsigned)m);
  count_launches(1);
  if (d_idx == 128)
    launch_kernel(true, decode_token_scores_kernel<128>, grid, 128, 0, s, ctx, capacity, B, m, blocks,
                  (const uint16_t*)q_new, (const uint16_t*)k_idx_cache, tkeys);
  else
    launch_kernel(true, decode_token_scores_kernel<64>, grid, 128, 0, s, ctx, capacity, B, m, blocks,
                  (const uint16_t*)q_new, (const uint16_t*)k_idx_cache, tkeys);
}

void launch_decode_combine(int batch, int64_t capacity, int32_t* ctx, int H, int d, int parts,
                           const float* Opart, const float* mpart, const float* lpart, void* O, cudaStream_t s) {
  if (batch == 0) return;
  count_launches(1);
  launch_kernel(true, decode_combine_kernel, unsigned(batch * H), d, 0, s, ctx, capacity, H, d, parts, Opart, mpart,
                lpart, (uint16_t*)O);
}

}  // namespace hsa
