// Decode-step helpers: append one token per sequence to the caller's caches
// (writing the block sum of a block the token completes) and advance the
// per-sequence lengths once the step's selection and attention are queued.
#include "kernels.cuh"

namespace hsa {

template <int DI, int DA>
__global__ void __launch_bounds__(128) decode_append_kernel(
    int64_t capacity, const int32_t* __restrict__ ctx, int B, uint16_t* __restrict__ k_idx_cache,
    uint16_t* __restrict__ K_cache, uint16_t* __restrict__ V_cache, float* __restrict__ ksum_cache,
    const uint16_t* __restrict__ k_idx_new, const uint16_t* __restrict__ K_new,
    const uint16_t* __restrict__ V_new) {
  const int64_t b = blockIdx.x;
  const int64_t t = ctx[b];
  if (t < 0 || t >= capacity) return;
  const int tid = threadIdx.x;
  const int64_t row = b * capacity + t;
  for (int e = tid; e < DI / 8; e += 128)
    reinterpret_cast<uint4*>(k_idx_cache + row * DI)[e] = reinterpret_cast<const uint4*>(k_idx_new + b * DI)[e];
  for (int e = tid; e < DA / 8; e += 128) {
    reinterpret_cast<uint4*>(K_cache + row * DA)[e] = reinterpret_cast<const uint4*>(K_new + b * DA)[e];
    reinterpret_cast<uint4*>(V_cache + row * DA)[e] = reinterpret_cast<const uint4*>(V_new + b * DA)[e];
  }
  if ((t + 1) % B != 0) return;
  // The token completes block t/B: its representative is the fp32 sum of
  // the block's rows (the new row taken from the input, the rest from the cache).
  const int64_t blk = t / B;
  for (int c = tid; c < DI; c += 128) {
    float s = 0.f;
    for (int64_t j = blk * B; j < t; ++j)
      s += __uint_as_float(uint32_t(k_idx_cache[(b * capacity + j) * DI + c]) << 16);
    s += __uint_as_float(uint32_t(k_idx_new[b * DI + c]) << 16);
    ksum_cache[(b * (capacity / B) + blk) * DI + c] = s;
  }
}

__global__ void decode_advance_kernel(int batch, int64_t capacity, int32_t* ctx) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < batch && ctx[b] >= 0 && ctx[b] < capacity) ctx[b] += 1;
}

void launch_decode_append(int batch, int64_t capacity, const int32_t* ctx, int B, int d_idx, int d,
                          void* k_idx_cache, void* K_cache, void* V_cache, float* ksum_cache,
                          const void* k_idx_new, const void* K_new, const void* V_new,
                          cudaStream_t s) {
  if (batch == 0) return;
  count_launches(1);
#define HSA_APPEND(DI, DA)                                                                      \
  decode_append_kernel<DI, DA><<<batch, 128, 0, s>>>(                                           \
      capacity, ctx, B, (uint16_t*)k_idx_cache, (uint16_t*)K_cache, (uint16_t*)V_cache,          \
      ksum_cache, (const uint16_t*)k_idx_new, (const uint16_t*)K_new, (const uint16_t*)V_new)
  if (d_idx == 128 && d == 128) HSA_APPEND(128, 128);
  else if (d_idx == 128) HSA_APPEND(128, 64);
  else if (d == 128) HSA_APPEND(64, 128);
  else HSA_APPEND(64, 64);
#undef HSA_APPEND
}

void launch_decode_advance(int batch, int64_t capacity, int32_t* ctx, cudaStream_t s) {
  if (batch == 0) return;
  count_launches(1);
  decode_advance_kernel<<<(batch + 127) / 128, 128, 0, s>>>(batch, capacity, ctx);
}

}  // namespace hsa
