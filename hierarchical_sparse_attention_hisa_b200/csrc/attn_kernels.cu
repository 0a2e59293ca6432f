// Sparse softmax attention over the kept tokens, multi-query (all H heads
// share the row's indices): O[i][h] = sum_j softmax_j(scale * Q[i][h] . K[j]) V[j]
// (the unchanged downstream attention of the HISA page's "drop-in
// replacement" paragraph; softmax(Q K^T / sqrt(d)) V as in the HiLS page's
// Step 4). CUDA-core kernel: one CTA per query row, keys streamed in chunks
// of 32 rows through shared memory, online softmax in the exp2 domain,
// fp32 accumulation, O rounded once to bf16.
#include "kernels.cuh"

namespace hsa {

template <int D, int HR>
__global__ void __launch_bounds__(128) sparse_attn_simple_kernel(
    RowMap rm, const uint16_t* __restrict__ Q, const uint16_t* __restrict__ K,
    const uint16_t* __restrict__ V, const int32_t* __restrict__ idx, int k, int H,
    float scale_log2, uint16_t* __restrict__ O) {
  griddep_wait();
  griddep_launch();
  constexpr int NT = 128, CH = 32, G = NT / D;
  extern __shared__ __align__(16) float sm[];
  float* Qs = sm;                       // [H][D]
  float* Ks = Qs + H * D;               // [CH][D+1]
  float* Vs = Ks + CH * (D + 1);        // [CH][D]
  float* P = Vs + CH * D;               // [H][CH]
  float* alpha = P + H * CH;            // [H]
  float* lsum = alpha + H;              // [H]
  float* mrun = lsum + H;               // [H]
  __shared__ int jrow[CH];

  const int64_t i = blockIdx.x;
  const int tid = threadIdx.x;
  const int c = tid % D, g = tid / D;
  uint16_t* out = O + i * int64_t(H) * D;
  if (!rm.valid(i)) {
    for (int e = tid; e < H * D; e += NT) out[e] = 0;
    return;
  }
  const int64_t row0 = rm.seq_row0(i);
  const int64_t limit = rm.ctx ? rm.capacity : rm.Lk;
  for (int e = tid; e < H * D; e += NT) Qs[e] = __uint_as_float(uint32_t(Q[i * int64_t(H) * D + e]) << 16);
  for (int h = tid; h < H; h += NT) { lsum[h] = 0.f; mrun[h] = -INFINITY; }
  float acc[HR];
#pragma unroll
  for (int r = 0; r < HR; ++r) acc[r] = 0.f;

  for (int j0 = 0; j0 < k; j0 += CH) {
    __syncthreads();
    if (tid < CH) {
      const int jj = j0 + tid;
      int64_t j = jj < k ? int64_t(idx[i * int64_t(k) + jj]) : -1;
      jrow[tid] = (j >= 0 && j < limit) ? int(j) : -1;
    }
    __syncthreads();
    for (int e = tid; e < CH * D / 8; e += NT) {
      const int r = e / (D / 8), cg = e % (D / 8);
      const int j = jrow[r];
      uint4 kv = make_uint4(0, 0, 0, 0), vv = make_uint4(0, 0, 0, 0);
      if (j >= 0) {
        kv = __ldg(reinterpret_cast<const uint4*>(K + (row0 + j) * D) + cg);
        vv = __ldg(reinterpret_cast<const uint4*>(V + (row0 + j) * D) + cg);
      }
      const uint32_t kw[4] = {kv.x, kv.y, kv.z, kv.w}, vw[4] = {vv.x, vv.y, vv.z, vv.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        Ks[r * (D + 1) + cg * 8 + 2 * q] = bf16_lo(kw[q]);
        Ks[r * (D + 1) + cg * 8 + 2 * q + 1] = bf16_hi(kw[q]);
        Vs[r * D + cg * 8 + 2 * q] = bf16_lo(vw[q]);
        Vs[r * D + cg * 8 + 2 * q + 1] = bf16_hi(vw[q]);
      }
    }
    __syncthreads();
    // scores, pre-multiplied by scale * log2(e)
    for (int p = tid; p < H * CH; p += NT) {
      const int h = p / CH, r = p % CH;
      float s = 0.f;
      for (int e = 0; e < D; ++e) s = __fmaf_rn(Qs[h * D + e], Ks[r * (D + 1) + e], s);
      P[p] = jrow[r] >= 0 ? s * scale_log2 : -INFINITY;
    }
    __syncthreads();
    for (int h = tid; h < H; h += NT) {
      float mx = mrun[h];
      for (int r = 0; r < CH; ++r) mx = fmaxf(mx, P[h * CH + r]);
      float a = 1.f, l = lsum[h];
      if (mx != -INFINITY) {
        a = exp2f(mrun[h] - mx);
        l *= a;
        for (int r = 0; r < CH; ++r) {
          const float pv = exp2f(P[h * CH + r] - mx);
          P[h * CH + r] = pv;
          l += pv;
        }
        mrun[h] = mx;
      } else {
        for (int r = 0; r < CH; ++r) P[h * CH + r] = 0.f;
      }
      alpha[h] = a;
      lsum[h] = l;
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < HR; ++r) {
      const int h = g + G * r;
      if (h < H) {
        float a = acc[r] * alpha[h];
        for (int q = 0; q < CH; ++q) a = __fmaf_rn(P[h * CH + q], Vs[q * D + c], a);
        acc[r] = a;
      }
    }
  }
  __syncthreads();
#pragma unroll
  for (int r = 0; r < HR; ++r) {
    const int h = g + G * r;
    if (h < H) {
      const float l = lsum[h];
      out[h * D + c] = uint16_t(f32_to_bf16_rn(l > 0.f ? acc[r] / l : 0.f));
    }
  }
}

template <int D, int HR>
static void launch_simple(RowMap rm, int64_t rows, const void* Q, const void* K, const void* V,
                          const int32_t* idx, int k, int H, float scale_log2, void* O,
                          cudaStream_t s, bool pdl) {
  const size_t smem = sizeof(float) * (size_t(H) * D + 32 * (D + 1) + 32 * D + size_t(H) * 32 + 3 * H);
  cudaFuncSetAttribute(sparse_attn_simple_kernel<D, HR>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       int(smem));
  launch_kernel(pdl, sparse_attn_simple_kernel<D, HR>, unsigned(rows), 128, smem, s, rm, (const uint16_t*)Q,
                (const uint16_t*)K, (const uint16_t*)V, idx, k, H, scale_log2, (uint16_t*)O);
}

void launch_sparse_attn_simple(RowMap rm, int64_t rows, const void* Q, const void* K, const void* V,
                               const int32_t* idx, int k, int H, int d, float scale, void* O,
                               cudaStream_t s, bool pdl) {
  if (rows == 0) return;
  count_launches(1);
  const float sl2 = scale * 1.4426950408889634f;
  if (d == 128) {
    if (H <= 16) launch_simple<128, 16>(rm, rows, Q, K, V, idx, k, H, sl2, O, s, pdl);
    else if (H <= 64) launch_simple<128, 64>(rm, rows, Q, K, V, idx, k, H, sl2, O, s, pdl);
    else launch_simple<128, 128>(rm, rows, Q, K, V, idx, k, H, sl2, O, s, pdl);
  } else {
    if (H <= 16) launch_simple<64, 8>(rm, rows, Q, K, V, idx, k, H, sl2, O, s, pdl);
    else if (H <= 64) launch_simple<64, 32>(rm, rows, Q, K, V, idx, k, H, sl2, O, s, pdl);
    else launch_simple<64, 64>(rm, rows, Q, K, V, idx, k, H, sl2, O, s, pdl);
  }
}

}  // namespace hsa
