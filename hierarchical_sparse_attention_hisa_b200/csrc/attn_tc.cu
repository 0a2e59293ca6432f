// Sparse softmax attention on tcgen05 tensor cores (sm_100a), multi-query:
// all H heads of a query share its k kept keys (the HISA page's "drop-in
// replacement" paragraph: the downstream sparse attention is unchanged;
// softmax(Q K^T / sqrt(d)) V as in the HiLS page's Step 4).
//
// Orientation: the kept keys, not the heads, are the MMA's M dimension, so
// every UMMA is a full 128-row tile whatever H is:
//   S^T[key][h] = Ktile[key][:] . Q[h][:]        (A = gathered K rows, K-major;
//                                                  B = the query's H x d block)
//   O^T[c][h]  += Vtile[key][c] . P^T[key][h]     (A = gathered V rows read
//                                                  MN-major; B = P^T, MN-major)
// Per CTA (persistent over queries) four warp roles run a pipeline:
//   warp 0     TMA producer: Q tile per query, K / V rows of each 128-key tile
//              fetched with tile::gather4 straight into 128B-swizzled smem;
//   warp 1     MMA issuer (one thread): S^T for tile g, then O^T for tile g-1;
//   warps 2-5  softmax + epilogue: thread = TMEM lane = key row of the tile.
// Softmax runs in the exp2 domain with a per-head running maximum that is
// only raised (and O^T, l rescaled) when a tile exceeds it by more than 2^8,
// so the cross-thread max reduction happens on the first tile of a query and
// rarely after. P is rounded to bf16 for the second MMA; accumulation is fp32.
#include "kernels.cuh"
#include "tc.cuh"

namespace hsa {

__device__ int g_attn_err;  // set when a bounded wait gives up

namespace {

using namespace tc;

constexpr int D = 128;       // head dim handled by this kernel
constexpr int TILE = 128;    // kept keys per MMA tile (the M dimension)
constexpr float kRescaleThreshold = 8.0f;  // log2 units

template <int HP, int NPW>
struct Cfg {
  static constexpr int NS = HP <= 32 ? 3 : 2;       // K/V pipeline stages
  static constexpr int HH = HP / 2;                 // heads per softmax warpgroup
  static constexpr int NWARPS = NPW + 1 + 8;        // producers, MMA issuer, 2 softmax warpgroups
  static constexpr int KV_BYTES = TILE * D * 2;     // one K or V tile: 32 KB
  static constexpr int Q_BYTES = HP * D * 2;        // one query's heads
  static constexpr int P_ROW = HP * 2;              // bytes of one P^T row (<= 128)
  static constexpr int P_BYTES = TILE * P_ROW;
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + NS * KV_BYTES;
  static constexpr int OFF_Q = OFF_V + NS * KV_BYTES;
  static constexpr int OFF_P = OFF_Q + 2 * Q_BYTES;
  static constexpr int SMEM = OFF_P + 2 * P_BYTES + 1024;  // + alignment slack
  static constexpr int TMEM_COLS = 4 * HP < 32 ? 32 : 4 * HP;
  static constexpr uint32_t P_SWZ = P_ROW == 128 ? kSw128 : P_ROW == 64 ? kSw64 : kSw32;
};

struct Bars {
  uint64_t kfull[3], kempty[3], vfull[3], vempty[3];
  uint64_t qfull[2], qempty[2], sfull[2], sempty[2], pfull[2], pempty[2], ofull[2], oempty[2];
  uint64_t done, group[2];
};

// Bounded wait that also gives up as soon as another role has reported a
// failure, so one lost arrival cannot keep any warp spinning for long.
HSA_DEV bool wait_bar(uint64_t* bar, uint32_t parity, bool& dead) {
  if (dead) return false;
  for (uint32_t it = 0; it < (1u << 24); ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 4095u) == 4095u && *(volatile int*)&g_attn_err) { dead = true; return false; }
  }
  atomicExch(&g_attn_err, 1);
  dead = true;
  return false;
}

// Warp-collective form: lane 0 polls, the outcome is broadcast, so every
// lane of the warp takes the same branch afterwards.
HSA_DEV bool wait_warp(uint64_t* bar, uint32_t parity, bool& dead) {
  bool ok = false;
  if ((threadIdx.x & 31) == 0) ok = wait_bar(bar, parity, dead);
  ok = __shfl_sync(kFull, ok ? 1 : 0, 0) != 0;
  __syncwarp();
  dead = !ok;
  return ok;
}

// Barrier over the four softmax warps on an mbarrier (count 4), bounded like
// every other wait; `phase` counts the barrier's completed phases.
HSA_DEV bool group_sync(uint64_t* bar, uint32_t& phase, bool& dead) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
  const bool ok = wait_warp(bar, phase & 1, dead);
  ++phase;
  return ok;
}

HSA_DEV float redux_max(float v) {
  float r;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}

// Sum of v[0..N) over the 32 lanes of a warp by halving exchanges; returns
// the number of distinct heads each lane ends with (NL) in v[0..NL), lane l
// holding heads l*NL .. l*NL+NL-1 when N >= 32, else head l / (32/N).
template <int N>
HSA_DEV void warp_transpose_sum(float (&v)[N]) {
  const int lane = threadIdx.x & 31;
  int n = N;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    if (n > 1) {
      const bool hi = lane & o;
      const int h = n / 2;
#pragma unroll
      for (int i = 0; i < N / 2; ++i) {
        if (i < h) {
          const float send = hi ? v[i] : v[i + h];
          const float keep = hi ? v[i + h] : v[i];
          v[i] = keep + __shfl_xor_sync(kFull, send, o);
        }
      }
      n = h;
    } else {
      v[0] += __shfl_xor_sync(kFull, v[0], o);
    }
  }
}
// Head index of value i after warp_transpose_sum<N> in lane `lane`.
template <int N>
HSA_DEV int transpose_head(int lane, int i) {
  if (N >= 32) return i + (N / 32) * lane;
  // n halves log2(N) times using lane bits 4, 3, ... ; the remaining low
  // lane bits only duplicate.
  constexpr int shift = (N == 16) ? 1 : (N == 8) ? 2 : (N == 4) ? 3 : (N == 2) ? 4 : 5;
  return lane >> shift;
}

// HH consecutive TMEM columns of this warp's 32 lanes into v (HH = 8, 16 or 32).
template <int HH>
HSA_DEV void tmem_ld_cols(uint32_t taddr, float (&v)[HH]) {
  if constexpr (HH == 8) {
    uint32_t r[8];
    tmem_ld8(taddr, r);
    tmem_wait_ld();
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] = __uint_as_float(r[e]);
  } else {
#pragma unroll
    for (int c0 = 0; c0 < HH; c0 += 16) {
      uint32_t r[16];
      tmem_ld16(taddr + c0, r);
      tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 16; ++e) v[c0 + e] = __uint_as_float(r[e]);
    }
  }
}
template <int HH>
HSA_DEV void tmem_st_cols(uint32_t taddr, const float (&v)[HH]) {
  if constexpr (HH == 8) {
    uint32_t r[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) r[e] = __float_as_uint(v[e]);
    tmem_st8(taddr, r);
  } else {
#pragma unroll
    for (int c0 = 0; c0 < HH; c0 += 16) {
      uint32_t r[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) r[e] = __float_as_uint(v[c0 + e]);
      tmem_st16(taddr + c0, r);
    }
  }
  tmem_wait_st();
}

template <int HP, int NPW>
__global__ void __launch_bounds__(32 * Cfg<HP, NPW>::NWARPS, 1) sparse_attn_tc_kernel(
    const __grid_constant__ CUtensorMap qmap, const uint16_t* __restrict__ K, const uint16_t* __restrict__ V,
    const int32_t* __restrict__ idx, int Lq, int Lk, int k, int H, float scale_log2, uint16_t* __restrict__ O) {
  using C = Cfg<HP, NPW>;
  constexpr int HH = C::HH;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) Bars bars;
  __shared__ uint32_t tmem_base;
  __shared__ int qinfo[2];
  __shared__ float red[4][HP];
  __shared__ float mh[HP];
  __shared__ float lsum[HP];
  __shared__ int vote[2][2][4];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(&bars.kfull[s], NPW * 32); mbar_init(&bars.kempty[s], 1);
      mbar_init(&bars.vfull[s], NPW * 32); mbar_init(&bars.vempty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars.qfull[b], 1); mbar_init(&bars.qempty[b], 1 + 8);
      mbar_init(&bars.sfull[b], 1); mbar_init(&bars.sempty[b], 8);
      mbar_init(&bars.pfull[b], 8); mbar_init(&bars.pempty[b], 1);
      mbar_init(&bars.ofull[b], 1); mbar_init(&bars.oempty[b], 8);
      mbar_init(&bars.group[b], 4);
    }
    mbar_init(&bars.done, 1);
    fence_barrier_init();
  }
  if (warp == NPW) { tmem_alloc(&tmem_base, C::TMEM_COLS); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;
  bool dead = false;

  if (warp < NPW) {
    // ------------------------------------------------------------ producers
    // Producer thread p copies the (row, 16-byte chunk) pairs p, p + 32*NPW, ...
    // of each K and V tile with cp.async into the 128B-swizzled layout UMMA reads.
    constexpr int PT = NPW * 32, PER = (TILE * 16 + PT - 1) / PT;
    const int p = threadIdx.x;
    if (p == 0) prefetch_tmap(&qmap);
    uint32_t g = 0, qn = 0;
    for (int q = blockIdx.x; q < Lq && !dead; q += gridDim.x, ++qn) {
      const int32_t* row = idx + int64_t(q) * k;
      int last = -1;  // tiles = ceil((last valid position + 1) / TILE)
      if ((k & 3) == 0) {
        const int4* row4 = reinterpret_cast<const int4*>(row);
#pragma unroll 4
        for (int p4 = lane; p4 < k / 4; p4 += 32) {
          const int4 v = __ldg(row4 + p4);
          if (v.x >= 0 && v.x < Lk) last = 4 * p4;
          if (v.y >= 0 && v.y < Lk) last = 4 * p4 + 1;
          if (v.z >= 0 && v.z < Lk) last = 4 * p4 + 2;
          if (v.w >= 0 && v.w < Lk) last = 4 * p4 + 3;
        }
      } else {
        for (int pp = lane; pp < k; pp += 32) {
          const int j = __ldg(row + pp);
          if (j >= 0 && j < Lk) last = pp;
        }
      }
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) last = max(last, __shfl_xor_sync(kFull, last, o));
      const int nt = (last + TILE) / TILE;
      const int qb = qn & 1;
      if (warp == 0) {
        if (!wait_warp(&bars.qempty[qb], ((qn >> 1) & 1) ^ 1, dead)) break;
        if (lane == 0) {
          qinfo[qb] = nt;
          mbar_arrive_expect_tx(&bars.qfull[qb], C::Q_BYTES);
          uint8_t* qt = sm + C::OFF_Q + qb * C::Q_BYTES;
          tma_load_2d(qt, &qmap, &bars.qfull[qb], 0, q * H);
          tma_load_2d(qt + HP * 128, &qmap, &bars.qfull[qb], 64, q * H);
        }
      }
      for (int i = 0; i < nt && !dead; ++i, ++g) {
        const int s = g % C::NS;
        const uint32_t ph = (g / C::NS) & 1;
        int64_t src[PER];
        uint32_t dst[PER];
#pragma unroll
        for (int u = 0; u < PER; ++u) {
          const int e = p + u * PT, r = (e >> 4) & (TILE - 1), c = e & 15;
          const int pos = i * TILE + r;
          const int j = (e < TILE * 16 && pos < k) ? __ldg(row + pos) : -1;
          src[u] = int64_t((j >= 0 && j < Lk) ? j : 0) * D + c * 8;
          dst[u] = (c >> 3) * (TILE * 128) + swz_offset(r, c & 7, 128);
        }
        if (!wait_warp(&bars.kempty[s], ph ^ 1, dead)) break;
        const uint32_t kt = smem_u32(sm + C::OFF_K + s * C::KV_BYTES);
#pragma unroll
        for (int u = 0; u < PER; ++u)
          if (p + u * PT < TILE * 16) cp_async16(kt + dst[u], K + src[u]);
        cp_async_arrive(&bars.kfull[s]);
        if (!wait_warp(&bars.vempty[s], ph ^ 1, dead)) break;
        const uint32_t vt = smem_u32(sm + C::OFF_V + s * C::KV_BYTES);
#pragma unroll
        for (int u = 0; u < PER; ++u)
          if (p + u * PT < TILE * 16) cp_async16(vt + dst[u], V + src[u]);
        cp_async_arrive(&bars.vfull[s]);
      }
    }
    cp_async_wait_all();  // every copy has landed before the CTA may exit
    if (warp == 0 && lane == 0) {
      bool d2 = false;
      for (uint32_t t = (qn >= 2 ? qn - 2 : 0); t < qn; ++t) wait_bar(&bars.qfull[t & 1], (t >> 1) & 1, d2);
    }
  } else if (warp == NPW) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t id_s = idesc_bf16(128, HP, false, false);
      constexpr uint32_t id_o = idesc_bf16(128, HP, true, true);
      uint32_t g = 0, qn = 0, oq = 0;
      struct Pend { uint32_t g, ob, oq; bool first, last, valid; } prev{0, 0, 0, false, false, false};
      auto issue_pv = [&](const Pend& t) {
        const int pb = t.g & 1, s = t.g % C::NS;
        if (!wait_bar(&bars.pfull[pb], (t.g >> 1) & 1, dead)) return;
        if (!wait_bar(&bars.vfull[s], (t.g / C::NS) & 1, dead)) return;
        if (t.first && !wait_bar(&bars.oempty[t.ob], ((t.oq >> 1) & 1) ^ 1, dead)) return;
        tc_fence_after();
        const uint32_t vbase = smem_u32(sm + C::OFF_V + s * C::KV_BYTES);
        const uint32_t pbase = smem_u32(sm + C::OFF_P + pb * C::P_BYTES);
#pragma unroll
        for (int ks = 0; ks < TILE / 16; ++ks) {
          const uint64_t a = smem_desc(vbase + ks * 2048, TILE * 128, 1024, kSw128);
          const uint64_t b = smem_desc(pbase + ks * 16 * C::P_ROW, 16384, 8 * C::P_ROW, C::P_SWZ);
          mma_bf16(tmem + 2 * HP + t.ob * HP, a, b, id_o, (t.first && ks == 0) ? 0u : 1u);
        }
        mma_commit(&bars.vempty[s]);
        mma_commit(&bars.pempty[pb]);
        if (t.last) mma_commit(&bars.ofull[t.ob]);
      };
      for (int q = blockIdx.x; q < Lq && !dead; q += gridDim.x, ++qn) {
        const int qb = qn & 1;
        if (!wait_bar(&bars.qfull[qb], (qn >> 1) & 1, dead)) break;
        const int nt = qinfo[qb];
        if (nt == 0) { mbar_arrive(&bars.qempty[qb]); continue; }
        const uint32_t ob = oq & 1;
        const uint32_t qbase = smem_u32(sm + C::OFF_Q + qb * C::Q_BYTES);
        for (int i = 0; i < nt && !dead; ++i, ++g) {
          const int s = g % C::NS, sb = g & 1;
          if (!wait_bar(&bars.kfull[s], (g / C::NS) & 1, dead)) break;
          if (!wait_bar(&bars.sempty[sb], ((g >> 1) & 1) ^ 1, dead)) break;
          tc_fence_after();
          const uint32_t kbase = smem_u32(sm + C::OFF_K + s * C::KV_BYTES);
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            const uint64_t a = smem_desc(kbase + (ks / 4) * TILE * 128 + (ks % 4) * 32, 16, 1024, kSw128);
            const uint64_t b = smem_desc(qbase + (ks / 4) * HP * 128 + (ks % 4) * 32, 16, 1024, kSw128);
            mma_bf16(tmem + sb * HP, a, b, id_s, ks > 0 ? 1u : 0u);
          }
          mma_commit(&bars.kempty[s]);
          mma_commit(&bars.sfull[sb]);
          if (i == nt - 1) mma_commit(&bars.qempty[qb]);
          if (prev.valid) issue_pv(prev);
          prev = Pend{g, ob, oq, i == 0, i == nt - 1, true};
        }
        ++oq;
      }
      if (prev.valid && !dead) issue_pv(prev);
      mma_commit(&bars.done);  // all issued MMAs complete before TMEM is released
      bool d2 = false;
      wait_bar(&bars.done, 0, d2);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax / epilogue
    // Two warpgroups; warpgroup wg owns heads [wg*HH, wg*HH + HH) of every tile.
    const int sw = warp - NPW - 1, wg = sw >> 2, wq = sw & 3;
    const int quad = warp & 3;              // TMEM lane quadrant this warp may access
    const int r = quad * 32 + lane;         // key row of the tile / dim row of O^T
    const int h0 = wg * HH;                 // first head of this warpgroup
    const uint32_t lane_addr = uint32_t(quad * 32) << 16;
    uint64_t* gbar = &bars.group[wg];
    uint32_t g = 0, qn = 0, oq = 0, gph = 0;
    for (int q = blockIdx.x; q < Lq && !dead; q += gridDim.x, ++qn) {
      const int qb = qn & 1;
      if (!wait_warp(&bars.qfull[qb], (qn >> 1) & 1, dead)) break;
      const int nt = qinfo[qb];
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.qempty[qb]);
      uint16_t* orow = O + int64_t(q) * H * D;
      if (nt == 0) {
        for (int h = h0; h < h0 + HH && h < H; ++h) orow[h * D + r] = 0;
        continue;
      }
      const uint32_t ob = oq & 1;
      const int32_t* irow = idx + int64_t(q) * k;
      float lp[HH];
#pragma unroll
      for (int h = 0; h < HH; ++h) lp[h] = 0.f;
      for (int i = 0; i < nt && !dead; ++i, ++g) {
        const int sb = g & 1;
        const int pos = i * TILE + r;
        const int j = pos < k ? __ldg(irow + pos) : -1;
        const bool valid = j >= 0 && j < Lk;
        if (!wait_warp(&bars.sfull[sb], (g >> 1) & 1, dead)) break;
        tc_fence_after();
        float x[HH];
        tmem_ld_cols<HH>(tmem + lane_addr + sb * HP + h0, x);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.sempty[sb]);
#pragma unroll
        for (int h = 0; h < HH; ++h) x[h] = (valid && h0 + h < H) ? x[h] * scale_log2 : -INFINITY;

        // Raise the running maxima only on the first tile, or when some
        // score exceeds its head's maximum by more than the threshold.
        bool need_max = (i == 0);
        if (!need_max) {
          bool mine = false;
#pragma unroll
          for (int h = 0; h < HH; ++h) mine |= x[h] > mh[h0 + h] + kRescaleThreshold;
          const bool any = __any_sync(kFull, mine);
          const uint32_t vb = gph & 1;
          if (lane == 0) vote[vb][wg][wq] = any;
          if (!group_sync(gbar, gph, dead)) break;
          need_max = vote[vb][wg][0] | vote[vb][wg][1] | vote[vb][wg][2] | vote[vb][wg][3];
        }
        if (need_max) {
#pragma unroll
          for (int h = 0; h < HH; ++h) {
            const float wm = redux_max(x[h]);
            if (lane == (h & 31)) red[wq][h0 + h] = wm;
          }
          if (!group_sync(gbar, gph, dead)) break;
          if (r < HH) {
            const int hh = h0 + r;
            const float tm = fmaxf(fmaxf(red[0][hh], red[1][hh]), fmaxf(red[2][hh], red[3][hh]));
            const float old = i == 0 ? -INFINITY : mh[hh];
            red[0][hh] = old;  // the previous maximum, for the rescale factors
            mh[hh] = fmaxf(old, tm);
          }
          if (!group_sync(gbar, gph, dead)) break;
          if (i > 0) {
            // rescale l and this warpgroup's O^T columns by 2^(old - new);
            // the previous tile's PV must have landed first.
            const uint32_t pg = g - 1;
            if (!wait_warp(&bars.pempty[pg & 1], (pg >> 1) & 1, dead)) break;
            tc_fence_after();
            float ov[HH];
            const uint32_t ta = tmem + lane_addr + 2 * HP + ob * HP + h0;
            tmem_ld_cols<HH>(ta, ov);
#pragma unroll
            for (int h = 0; h < HH; ++h) {
              const float o = red[0][h0 + h], n = mh[h0 + h];
              const float a = (o == -INFINITY || n == -INFINITY) ? (o == n ? 1.f : 0.f) : exp2f(o - n);
              lp[h] *= a;
              ov[h] *= a;
            }
            tmem_st_cols<HH>(ta, ov);
            // red[0] holds the old maxima until every thread has read them
            if (!group_sync(gbar, gph, dead)) break;
          }
        }
        // probabilities, partial row sums, this warpgroup's part of the P^T row
        const int pb = g & 1;
        if (!wait_warp(&bars.pempty[pb], ((g >> 1) & 1) ^ 1, dead)) break;
        uint8_t* prow = sm + C::OFF_P + pb * C::P_BYTES;
#pragma unroll
        for (int c = 0; c < HH / 8; ++c) {
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int a0 = c * 8 + 2 * e;
            const float p0 = x[a0] == -INFINITY ? 0.f : exp2f(x[a0] - mh[h0 + a0]);
            const float p1 = x[a0 + 1] == -INFINITY ? 0.f : exp2f(x[a0 + 1] - mh[h0 + a0 + 1]);
            lp[a0] += p0;
            lp[a0 + 1] += p1;
            w[e] = pack_bf16x2(p0, p1);
          }
          *reinterpret_cast<uint4*>(prow + swz_offset(r, h0 / 8 + c, C::P_ROW)) = make_uint4(w[0], w[1], w[2], w[3]);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.pfull[pb]);
      }
      if (dead) break;
      // ---- epilogue: row sums, normalise O^T, write O[q][h][r] for this warpgroup's heads
      warp_transpose_sum<HH>(lp);
      constexpr int NL = HH >= 32 ? HH / 32 : 1;
      if (HH >= 32 || (lane & ((32 / HH) - 1)) == 0) {
#pragma unroll
        for (int e = 0; e < NL; ++e) red[wq][h0 + transpose_head<HH>(lane, e)] = lp[e];
      }
      if (!group_sync(gbar, gph, dead)) break;
      if (r < HH) lsum[h0 + r] = red[0][h0 + r] + red[1][h0 + r] + red[2][h0 + r] + red[3][h0 + r];
      if (!group_sync(gbar, gph, dead)) break;
      if (!wait_warp(&bars.ofull[ob], (oq >> 1) & 1, dead)) break;
      tc_fence_after();
      float ov[HH];
      tmem_ld_cols<HH>(tmem + lane_addr + 2 * HP + ob * HP + h0, ov);
#pragma unroll
      for (int h = 0; h < HH; ++h) {
        if (h0 + h < H) {
          const float l = lsum[h0 + h];
          orow[(h0 + h) * D + r] = uint16_t(f32_to_bf16_rn(l > 0.f ? ov[h] / l : 0.f));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.oempty[ob]);
      // lsum / red are reused by the next query only after the warpgroup is done
      if (!group_sync(gbar, gph, dead)) break;
      ++oq;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == NPW) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// 7 producer warps + 1 MMA warp + 8 softmax warps = 16 warps, 4 per SM
// sub-partition, which leaves 128 registers per thread.
constexpr int kProducerWarps = 7;

template <int HP>
bool launch_hp(const void* Q, const void* K, const void* V, const int32_t* idx, int Lq, int Lk, int k,
               int H, float scale_log2, void* O, cudaStream_t s) {
  CUtensorMap qm;
  if (!make_tmap_2d(&qm, Q, uint64_t(Lq) * H, D, HP)) return false;
  using C = Cfg<HP, kProducerWarps>;
  auto kern = sparse_attn_tc_kernel<HP, kProducerWarps>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) != cudaSuccess)
    return false;
  const int grid = Lq < num_sms() ? Lq : num_sms();
  kern<<<grid, 32 * C::NWARPS, C::SMEM, s>>>(qm, static_cast<const uint16_t*>(K), static_cast<const uint16_t*>(V),
                                             idx, Lq, Lk, k, H, scale_log2, static_cast<uint16_t*>(O));
  return true;
}

}  // namespace

bool tc_attn_supported(int H, int d, int64_t Lq, int64_t Lk) {
  const int hp = H <= 16 ? 16 : H <= 32 ? 32 : 64;
  // the Q box (hp rows) must fit inside the [Lq*H][d] tensor map
  return d == 128 && H >= 1 && H <= 64 && Lq * H >= hp && Lq * H < (int64_t(1) << 31) &&
         Lk < (int64_t(1) << 31);
}

bool launch_sparse_attn_tc(int64_t Lq, const void* Q, const void* K, const void* V, const int32_t* idx,
                           int64_t Lk, int k, int H, float scale, void* O, cudaStream_t s) {
  if (Lq == 0) return true;
  count_launches(1);
  const float sl2 = scale * 1.4426950408889634f;
  const int L = int(Lq), LK = int(Lk);
  if (H <= 16) return launch_hp<16>(Q, K, V, idx, L, LK, k, H, sl2, O, s);
  if (H <= 32) return launch_hp<32>(Q, K, V, idx, L, LK, k, H, sl2, O, s);
  return launch_hp<64>(Q, K, V, idx, L, LK, k, H, sl2, O, s);
}

}  // namespace hsa
