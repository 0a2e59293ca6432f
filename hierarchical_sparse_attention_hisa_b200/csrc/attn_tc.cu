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
// Per CTA (persistent over queries) the warp roles form a pipeline:
//   warps 0..6   producers: Q tile per query by TMA; the K / V rows of each
//                128-key tile by cp.async straight into the 128B-swizzled
//                layout UMMA reads (row gathers through the LSU sustain far
//                more bandwidth than TMA's four-row gathers);
//   warp 7       MMA issuer (one thread): S^T of tile g, then O^T of tile g-1;
//   warps 8..23  four softmax warpgroups, warpgroup w owning heads
//                [w*H/4, (w+1)*H/4): thread = TMEM lane = key row of the tile.
// Softmax runs in the exp2 domain with a per-head running maximum that is
// only raised (and O^T, l rescaled) when a tile exceeds it by more than 2^8,
// so the cross-thread max reduction happens on a query's first tile and
// rarely after; the per-tile check is one hardware barrier reduction. P is
// rounded to bf16 for the second MMA; accumulation is fp32.
//
// A barrier probe in the MMA-issuing thread costs about as much as an MMA
// when MMAs are queued, so with two stages that thread waits on one barrier
// per MMA group: "K tile landed and S buffer read" before S, "P written and V
// tile landed" before PV, each counting the arrivals of both producers.
//
// Every mbarrier wait is bounded. Within a softmax warpgroup all four warps
// take the same sequence of named barriers: a failed wait is folded into the
// next barrier reduction, after which the whole warpgroup leaves together.
#include "kernels.cuh"
#include "tc.cuh"

namespace hsa {

__device__ int g_attn_err;  // set when a bounded wait gives up

namespace {

using namespace tc;

constexpr int D = 128;       // head dim handled by this kernel
constexpr int TILE = 128;    // kept keys per MMA tile (the M dimension)
constexpr int NWG = 4;       // softmax warpgroups
constexpr float kRescaleThreshold = 8.0f;  // log2 units

template <int HP, int NPW>
struct Cfg {
  static constexpr int NS = HP <= 32 ? 3 : 2;       // K/V pipeline stages
  static constexpr int HH = HP / NWG;               // heads per softmax warpgroup
  static constexpr int NSW = 4 * NWG;               // softmax warps
  static constexpr int NWARPS = NPW + 1 + NSW;
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
  // two stages: sgo = K tile landed + S buffer read, pgo = P tile written + V tile landed
  uint64_t sgo[2], pgo[2];
  uint64_t done;
};

}  // namespace

// Work description of one launch. Query q's kept indices are idx[q][0..k);
// its K/V rows start at row q * kv_stride (0: one K/V shared by all queries).
// Each query is cut into items_per_query parts of tiles_per_item 128-key
// tiles; with one part per query the kernel writes normalised O, otherwise
// every part w = q * items_per_query + s writes its unnormalised O^T, running
// maximum and row sum for a later combination.
struct AttnArgs {
  const int32_t* idx;
  int Lq, Lk, k, H;
  float scale_log2;
  int64_t kv_stride;
  int items_per_query, tiles_per_item;
  uint16_t* O;
  float *Opart, *mpart, *lpart;  // [items][H][D], [items][H], [items][H]
};

namespace {

// Bounded wait that also gives up as soon as another role has reported a
// failure, so one lost arrival cannot keep any warp spinning for long.
HSA_DEV bool wait_bar(uint64_t* bar, uint32_t parity, bool& dead) {
  if (dead) return false;
  if (mbar_wait_bounded(bar, parity, &g_attn_err)) return true;
  dead = true;
  return false;
}
// Warp form for the producers: lane 0 polls, the outcome is broadcast.
HSA_DEV bool wait_warp(uint64_t* bar, uint32_t parity, bool& dead) {
  bool ok = false;
  if ((threadIdx.x & 31) == 0) ok = wait_bar(bar, parity, dead);
  ok = __shfl_sync(kFull, ok ? 1 : 0, 0) != 0;
  dead = !ok;
  return ok;
}
// Warp form for the softmax warps: every lane polls, the result is the
// warp-wide AND (so warp-collective tcgen05 loads stay converged).
HSA_DEV bool wait_all(uint64_t* bar, uint32_t parity, bool dead) {
  bool d = dead;
  const bool ok = wait_bar(bar, parity, d);
  return __all_sync(kFull, ok);
}

// Named barrier `id` over one softmax warpgroup (128 threads).
HSA_DEV void wg_sync(int id) { asm volatile("bar.sync %0, 128;" ::"r"(id) : "memory"); }
HSA_DEV bool wg_or(int id, bool v) {
  uint32_t out;
  asm volatile(
      "{\n .reg .pred a, b;\n setp.ne.u32 a, %2, 0;\n bar.red.or.pred b, %1, 128, a;\n selp.u32 %0, 1, 0, b;\n}"
      : "=r"(out)
      : "r"(id), "r"(uint32_t(v))
      : "memory");
  return out != 0;
}

HSA_DEV float redux_max(float v) {
  float r;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}

// Sum of v[0..N) over the 32 lanes of a warp by halving exchanges. Lane l
// ends with the sums of heads transpose_head<N>(l, e), e < max(N/32, 1).
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
template <int N>
HSA_DEV int transpose_head(int lane, int i) {
  if (N >= 32) return i + (N / 32) * lane;
  // the halvings consume lane bits 4, 3, ...; the remaining low bits duplicate
  constexpr int shift = (N == 16) ? 1 : (N == 8) ? 2 : (N == 4) ? 3 : (N == 2) ? 4 : 5;
  return lane >> shift;
}

// N consecutive 32-bit TMEM columns of this warp's 32 lanes (N = 4, 8, 16).
template <int N>
HSA_DEV void tmem_ld_cols(uint32_t taddr, float (&v)[N]) {
  uint32_t r[N];
  if constexpr (N == 4) tmem_ld4(taddr, r);
  else if constexpr (N == 8) tmem_ld8(taddr, r);
  else tmem_ld16(taddr, r);
  tmem_wait_ld();
#pragma unroll
  for (int e = 0; e < N; ++e) v[e] = __uint_as_float(r[e]);
}
template <int N>
HSA_DEV void tmem_st_cols(uint32_t taddr, const float (&v)[N]) {
  uint32_t r[N];
#pragma unroll
  for (int e = 0; e < N; ++e) r[e] = __float_as_uint(v[e]);
  if constexpr (N == 4) tmem_st4(taddr, r);
  else if constexpr (N == 8) tmem_st8(taddr, r);
  else tmem_st16(taddr, r);
  tmem_wait_st();
}

template <int HP, int NPW>
__global__ void __launch_bounds__(32 * Cfg<HP, NPW>::NWARPS, 1) sparse_attn_tc_kernel(
    const __grid_constant__ CUtensorMap qmap, const uint16_t* __restrict__ K, const uint16_t* __restrict__ V,
    const AttnArgs a) {
  using C = Cfg<HP, NPW>;
  const int32_t* __restrict__ idx = a.idx;
  const int Lk = a.Lk, k = a.k, H = a.H;
  const float scale_log2 = a.scale_log2;
  const int ipq = a.items_per_query, tpi = a.tiles_per_item;
  const int n_items = a.Lq * ipq;
  constexpr int HH = C::HH;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) Bars bars;
  __shared__ uint32_t tmem_base;
  __shared__ int qinfo[2][2];  // per Q buffer: first tile, tile count
  __shared__ float red[4][HP];
  __shared__ float mh[HP];
  __shared__ float lsum[HP];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(&bars.kfull[s], NPW * 32); mbar_init(&bars.kempty[s], 1);
      mbar_init(&bars.vfull[s], NPW * 32); mbar_init(&bars.vempty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars.qfull[b], 1); mbar_init(&bars.qempty[b], 1 + C::NSW);
      mbar_init(&bars.sfull[b], 1); mbar_init(&bars.sempty[b], C::NSW);
      mbar_init(&bars.pfull[b], C::NSW); mbar_init(&bars.pempty[b], 1);
      mbar_init(&bars.sgo[b], NPW * 32 + C::NSW); mbar_init(&bars.pgo[b], NPW * 32 + C::NSW);
      // each S buffer starts out read: credit the softmax arrivals of its first use
      for (int u = 0; u < C::NSW; ++u) mbar_arrive(&bars.sgo[b]);
      mbar_init(&bars.ofull[b], 1); mbar_init(&bars.oempty[b], C::NSW);
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
  // barrier set-up and the TMEM allocation above touch no global memory, so
  // under a programmatic dependent launch they overlap the previous kernel
  griddep_wait();
  griddep_launch();

  if (warp < NPW) {
    // ------------------------------------------------------------ producers
    // Producer thread p copies the (row, 16-byte chunk) pairs p, p + 32*NPW, ...
    // of each K and V tile with cp.async into the 128B-swizzled layout.
    constexpr int PT = NPW * 32, PER = (TILE * 16 + PT - 1) / PT;
    const int p = threadIdx.x;
    if (p == 0) prefetch_tmap(&qmap);
    // The tile count of a query needs its last valid index position: the
    // row is searched backwards 128 entries at a time, and the last 128
    // entries of the next query's row are fetched one query ahead, so the
    // usual case (a valid tail) costs no exposed load latency.
    const bool vec = (k & 3) == 0 && k >= 128;
    const int s0 = vec ? k - 128 : 0;  // start of the last 128-entry window
    auto tail_window = [&](int q) -> int4 {
      return vec ? __ldg(reinterpret_cast<const int4*>(idx + int64_t(q) * k + s0) + lane) : make_int4(-1, -1, -1, -1);
    };
    int4 pre = blockIdx.x < n_items ? tail_window(blockIdx.x / ipq) : make_int4(-1, -1, -1, -1);
    uint32_t g = 0, qn = 0;
    for (int w = blockIdx.x; w < n_items && !dead; w += gridDim.x, ++qn) {
      const int q = w / ipq, part = w - q * ipq;
      const int32_t* row = idx + int64_t(q) * k;
      const uint4* Kq = reinterpret_cast<const uint4*>(K + int64_t(q) * a.kv_stride * D);
      const uint4* Vq = reinterpret_cast<const uint4*>(V + int64_t(q) * a.kv_stride * D);
      const int4 win = pre;
      if (w + int(gridDim.x) < n_items) pre = tail_window((w + gridDim.x) / ipq);
      int last = -1;  // tiles = ceil((last valid position + 1) / TILE)
      if (vec) {
        if (win.x >= 0 && win.x < Lk) last = s0 + 4 * lane;
        if (win.y >= 0 && win.y < Lk) last = s0 + 4 * lane + 1;
        if (win.z >= 0 && win.z < Lk) last = s0 + 4 * lane + 2;
        if (win.w >= 0 && win.w < Lk) last = s0 + 4 * lane + 3;
      }
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) last = max(last, __shfl_xor_sync(kFull, last, o));
      for (int c0 = (vec ? s0 : k) - 32; last < 0 && c0 > -32; c0 -= 32) {  // backwards, 32 at a time
        const int pp = c0 + lane;
        const int j = pp >= 0 ? __ldg(row + pp) : -1;
        const unsigned v = __ballot_sync(kFull, j >= 0 && j < Lk);
        if (v) last = c0 + 31 - __clz(v);
      }
      const int t0 = part * tpi;                                  // this item's tiles
      const int nt = max(0, min((last + TILE) / TILE, t0 + tpi) - t0);
      const int qb = qn & 1;
      if (warp == 0) {
        if (!wait_warp(&bars.qempty[qb], ((qn >> 1) & 1) ^ 1, dead)) break;
        if (lane == 0) {
          qinfo[qb][0] = t0;
          qinfo[qb][1] = nt;
          mbar_arrive_expect_tx(&bars.qfull[qb], C::Q_BYTES);
          uint8_t* qt = sm + C::OFF_Q + qb * C::Q_BYTES;
          tma_load_2d(qt, &qmap, &bars.qfull[qb], 0, q * H);
          tma_load_2d(qt + HP * 128, &qmap, &bars.qfull[qb], 64, q * H);
        }
      }
      for (int i = 0; i < nt && !dead; ++i, ++g) {
        const int s = g % C::NS;
        const uint32_t ph = (g / C::NS) & 1;
        int jr[PER];
        uint32_t dst[PER];
#pragma unroll
        for (int u = 0; u < PER; ++u) {
          const int e = p + u * PT, r = (e >> 4) & (TILE - 1), c = e & 15;
          const int pos = (t0 + i) * TILE + r;
          const int j = (e < TILE * 16 && pos < k) ? __ldg(row + pos) : -1;
          jr[u] = ((j >= 0 && j < Lk) ? j : 0) * (D / 8) + c;   // 16-byte units
          dst[u] = (c >> 3) * (TILE * 128) + swz_offset(r, c & 7, 128);
        }
        // with two stages, a K stage is free once S of the tile two back is
        // done (sfull), a V stage once its PV is done (pempty)
        if (!wait_warp(C::NS == 2 ? &bars.sfull[s] : &bars.kempty[s], ph ^ 1, dead)) break;
        const uint32_t kt = smem_u32(sm + C::OFF_K + s * C::KV_BYTES);
#pragma unroll
        for (int u = 0; u < PER; ++u)
          if (p + u * PT < TILE * 16) cp_async16(kt + dst[u], Kq + jr[u]);
        cp_async_arrive(C::NS == 2 ? &bars.sgo[s] : &bars.kfull[s]);
        if (!wait_warp(C::NS == 2 ? &bars.pempty[s] : &bars.vempty[s], ph ^ 1, dead)) break;
        const uint32_t vt = smem_u32(sm + C::OFF_V + s * C::KV_BYTES);
#pragma unroll
        for (int u = 0; u < PER; ++u)
          if (p + u * PT < TILE * 16) cp_async16(vt + dst[u], Vq + jr[u]);
        cp_async_arrive(C::NS == 2 ? &bars.pgo[s] : &bars.vfull[s]);
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
        if constexpr (C::NS == 2) {
          // one wait per tile: P written and V landed
          if (!wait_bar(&bars.pgo[pb], (t.g >> 1) & 1, dead)) return;
        } else {
          if (!wait_bar(&bars.pfull[pb], (t.g >> 1) & 1, dead)) return;
          if (!wait_bar(&bars.vfull[s], (t.g / C::NS) & 1, dead)) return;
        }
        if (t.first && !wait_bar(&bars.oempty[t.ob], ((t.oq >> 1) & 1) ^ 1, dead)) return;
        // the V rows landed by cp.async (generic proxy) are read by the MMA
        // (async proxy): order them across proxies after the acquire above
        fence_proxy_async_smem();
        tc_fence_after();
        const uint64_t a0 = smem_desc(smem_u32(sm + C::OFF_V + s * C::KV_BYTES), TILE * 128, 1024, kSw128);
        const uint64_t b0 = smem_desc(smem_u32(sm + C::OFF_P + pb * C::P_BYTES), 16384, 8 * C::P_ROW, C::P_SWZ);
        const uint32_t d = tmem + 2 * HP + t.ob * HP;
        const uint32_t alo = uint32_t(a0), ahi = uint32_t(a0 >> 32), blo = uint32_t(b0), bhi = uint32_t(b0 >> 32);
#pragma unroll
        for (int ks = 0; ks < TILE / 16; ++ks)
          mma_bf16_split(d, alo + ((ks * 2048) >> 4), ahi, blo + ((ks * 16 * C::P_ROW) >> 4), bhi, id_o,
                         (t.first && ks == 0) ? 0u : 1u);
        if (C::NS != 2) mma_commit(&bars.vempty[s]);
        mma_commit(&bars.pempty[pb]);
        if (t.last) mma_commit(&bars.ofull[t.ob]);
      };
      for (int w = blockIdx.x; w < n_items && !dead; w += gridDim.x, ++qn) {
        const int qb = qn & 1;
        if (!wait_bar(&bars.qfull[qb], (qn >> 1) & 1, dead)) break;
        const int nt = qinfo[qb][1];
        if (nt == 0) { mbar_arrive(&bars.qempty[qb]); continue; }
        const uint32_t ob = oq & 1;
        const uint64_t qd0 = smem_desc(smem_u32(sm + C::OFF_Q + qb * C::Q_BYTES), 16, 1024, kSw128);
        const uint32_t qlo = uint32_t(qd0), qhi = uint32_t(qd0 >> 32);
        for (int i = 0; i < nt && !dead; ++i, ++g) {
          const int s = g % C::NS, sb = g & 1;
          if constexpr (C::NS == 2) {
            // one wait per tile: K landed and the S buffer read by the softmax
            if (!wait_bar(&bars.sgo[sb], (g >> 1) & 1, dead)) break;
          } else {
            if (!wait_bar(&bars.kfull[s], (g / C::NS) & 1, dead)) break;
            if (!wait_bar(&bars.sempty[sb], ((g >> 1) & 1) ^ 1, dead)) break;
          }
          fence_proxy_async_smem();  // K rows landed by cp.async, read by the MMA
          tc_fence_after();
          const uint64_t kd0 = smem_desc(smem_u32(sm + C::OFF_K + s * C::KV_BYTES), 16, 1024, kSw128);
          const uint32_t klo = uint32_t(kd0), khi = uint32_t(kd0 >> 32);
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks)
            mma_bf16_split(tmem + sb * HP, klo + (((ks / 4) * TILE * 128 + (ks % 4) * 32) >> 4), khi,
                           qlo + (((ks / 4) * HP * 128 + (ks % 4) * 32) >> 4), qhi, id_s, ks > 0 ? 1u : 0u);
          if (C::NS != 2) mma_commit(&bars.kempty[s]);
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
    const int sw = warp - NPW - 1, wg = sw >> 2;
    const int bar_id = 1 + wg;
    const int quad = warp & 3;              // TMEM lane quadrant this warp may access
    const int wq = quad;                    // slot of this warp in the warpgroup's scratch rows
    const int r = quad * 32 + lane;         // key row of the tile / dim row of O^T
    const int h0 = wg * HH;                 // first head of this warpgroup
    const uint32_t lane_addr = uint32_t(quad * 32) << 16;
    uint32_t g = 0, qn = 0, oq = 0;
    for (int w = blockIdx.x; w < n_items; w += gridDim.x, ++qn) {
      const int q = w / ipq;
      const int qb = qn & 1;
      const bool okq = wait_all(&bars.qfull[qb], (qn >> 1) & 1, dead);
      if (wg_or(bar_id, !okq || dead)) { dead = true; break; }
      const int t0 = qinfo[qb][0], nt = qinfo[qb][1];
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.qempty[qb]);
      uint16_t* orow = a.O ? a.O + int64_t(q) * H * D : nullptr;
      if (nt == 0) {
        if (orow) {
#pragma unroll
          for (int h = 0; h < HH; ++h)
            if (h0 + h < H) orow[(h0 + h) * D + r] = 0;
        } else if (r < HH && h0 + r < H) {  // an empty part: no weight in the combination
          a.mpart[int64_t(w) * H + h0 + r] = -INFINITY;
          a.lpart[int64_t(w) * H + h0 + r] = 0.f;
        }
        continue;
      }
      const uint32_t ob = oq & 1;
      const int32_t* irow = idx + int64_t(q) * k;
      // m: running maximum per head (log2 units), or 0 while the head has
      // seen no valid key (its scores so far are all -inf, so 2^(x - 0) = 0);
      // `complete`: every real head of this warpgroup has a finite maximum.
      float lp[HH], m[HH];
#pragma unroll
      for (int h = 0; h < HH; ++h) { lp[h] = 0.f; m[h] = 0.f; }
      bool complete = false;
      bool quit = false;
      for (int i = 0; i < nt; ++i, ++g) {
        const int sb = g & 1;
        const int pos = (t0 + i) * TILE + r;
        const int j = pos < k ? __ldg(irow + pos) : -1;
        const bool valid = j >= 0 && j < Lk;
        const bool oks = wait_all(&bars.sfull[sb], (g >> 1) & 1, dead);
        float x[HH];
        if (oks) {
          tc_fence_after();
          tmem_ld_cols<HH>(tmem + lane_addr + sb * HP + h0, x);
        }
        tc_fence_before();
        __syncwarp();
        // (with two stages this arrival counts toward the buffer's next use)
        if (lane == 0) mbar_arrive(C::NS == 2 ? &bars.sgo[sb] : &bars.sempty[sb]);
        // x becomes the exponent scale * s - m; a row without a valid key and
        // padded heads get -inf (no weight)
        const bool live = oks && valid;
        float tmax = -INFINITY;
#pragma unroll
        for (int h = 0; h < HH; ++h) {
          x[h] = fmaf(x[h], scale_log2, -m[h]);
          tmax = fmaxf(tmax, x[h]);
        }
        if (!live || h0 + HH > H) {
          tmax = -INFINITY;
#pragma unroll
          for (int h = 0; h < HH; ++h) {
            if (!live || h0 + h >= H) x[h] = -INFINITY;
            tmax = fmaxf(tmax, x[h]);
          }
        }
        const bool mine = tmax > kRescaleThreshold || !complete;
        dead = dead || !oks;
        if (wg_or(bar_id, i == 0 || mine || dead)) {
          if (wg_or(bar_id, dead)) { quit = true; break; }
          // raise the running maxima of this warpgroup's heads to cover the tile
#pragma unroll
          for (int h = 0; h < HH; ++h) {
            const float wm = redux_max(x[h] + m[h]);  // the tile's scaled scores
            if (lane == (h & 31)) red[wq][h0 + h] = wm;
          }
          wg_sync(bar_id);
          if (r < HH) {
            const int hh = h0 + r;
            const float tm = fmaxf(fmaxf(red[0][hh], red[1][hh]), fmaxf(red[2][hh], red[3][hh]));
            const float old = i == 0 ? -INFINITY : mh[hh];
            red[0][hh] = old;  // the previous maximum, for the rescale factors
            mh[hh] = fmaxf(old, tm);
          }
          wg_sync(bar_id);
          bool all = true;
#pragma unroll
          for (int h = 0; h < HH; ++h) {
            const float n = mh[h0 + h];
            const float mn = n == -INFINITY ? 0.f : n;
            x[h] += m[h] - mn;  // re-centre the exponents on the new maximum
            m[h] = mn;
            all = all && (n != -INFINITY || h0 + h >= H);
          }
          complete = all;
          if (i > 0) {
            // rescale l and this warpgroup's O^T columns; the previous
            // tile's PV must have landed first
            const uint32_t pg = g - 1;
            const bool okp = wait_all(&bars.pempty[pg & 1], (pg >> 1) & 1, dead);
            dead = dead || !okp;
            if (okp) {
              tc_fence_after();
              float ov[HH];
              const uint32_t ta = tmem + lane_addr + 2 * HP + ob * HP + h0;
              tmem_ld_cols<HH>(ta, ov);
#pragma unroll
              for (int h = 0; h < HH; ++h) {
                // o = -inf: nothing accumulated yet (factor 0); n = -inf: no valid key yet
                const float o = red[0][h0 + h], n = mh[h0 + h];
                const float a = n == -INFINITY ? 1.f : ex2(o - n);
                lp[h] *= a;
                ov[h] *= a;
              }
              tmem_st_cols<HH>(ta, ov);
            }
          }
          wg_sync(bar_id);  // red[0] holds the old maxima until everyone has read them
        }
        // probabilities, partial row sums, this warpgroup's part of the P^T row
        const int pb = g & 1;
        const bool okw = wait_all(&bars.pempty[pb], ((g >> 1) & 1) ^ 1, dead);
        dead = dead || !okw;
        uint32_t w[(HH + 1) / 2];
#pragma unroll
        for (int e = 0; e < HH / 2; ++e) {
          const float p0 = ex2(x[2 * e]), p1 = ex2(x[2 * e + 1]);
          lp[2 * e] += p0;
          lp[2 * e + 1] += p1;
          w[e] = cvt_bf16x2(p0, p1);
        }
        if (okw) {
          uint8_t* prow = sm + C::OFF_P + pb * C::P_BYTES;
          if constexpr (HH >= 8) {
#pragma unroll
            for (int c = 0; c < HH / 8; ++c)
              *reinterpret_cast<uint4*>(prow + swz_offset(r, h0 / 8 + c, C::P_ROW)) =
                  make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
          } else {
            *reinterpret_cast<uint2*>(prow + swz_offset(r, h0 / 8, C::P_ROW) + (h0 % 8) * 2) = make_uint2(w[0], w[1]);
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(C::NS == 2 ? &bars.pgo[pb] : &bars.pfull[pb]);
      }
      if (quit) break;
      // ---- epilogue: row sums, normalise O^T, write O[q][h][r] for this warpgroup's heads
      warp_transpose_sum<HH>(lp);
      constexpr int NL = HH >= 32 ? HH / 32 : 1;
      if (HH >= 32 || (lane & ((32 / HH) - 1)) == 0) {
#pragma unroll
        for (int e = 0; e < NL; ++e) red[wq][h0 + transpose_head<HH>(lane, e)] = lp[e];
      }
      wg_sync(bar_id);
      if (r < HH) lsum[h0 + r] = red[0][h0 + r] + red[1][h0 + r] + red[2][h0 + r] + red[3][h0 + r];
      wg_sync(bar_id);
      const bool oko = wait_all(&bars.ofull[ob], (oq >> 1) & 1, dead);
      if (oko) {
        tc_fence_after();
        float ov[HH];
        tmem_ld_cols<HH>(tmem + lane_addr + 2 * HP + ob * HP + h0, ov);
        if (orow) {
#pragma unroll
          for (int h = 0; h < HH; ++h) {
            if (h0 + h < H) {
              const float l = lsum[h0 + h];
              orow[(h0 + h) * D + r] = uint16_t(f32_to_bf16_rn(l > 0.f ? ov[h] / l : 0.f));
            }
          }
        } else {
          // one part of a split query: unnormalised O^T, running maximum, row sum
          float* op = a.Opart + int64_t(w) * H * D;
#pragma unroll
          for (int h = 0; h < HH; ++h)
            if (h0 + h < H) op[(h0 + h) * D + r] = ov[h];
          if (r < HH && h0 + r < H) {
            a.mpart[int64_t(w) * H + h0 + r] = mh[h0 + r];
            a.lpart[int64_t(w) * H + h0 + r] = lsum[h0 + r];
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.oempty[ob]);
      // also keeps red / lsum untouched until the whole warpgroup is done
      if (wg_or(bar_id, dead || !oko)) { dead = true; break; }
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

// 7 producer warps + 1 MMA warp + 16 softmax warps = 24 warps (6 per SM
// sub-partition, 80 registers per thread).
constexpr int kProducerWarps = 7;

template <int HP>
bool launch_hp(const void* Q, const void* K, const void* V, const AttnArgs& a, cudaStream_t s, bool pdl) {
  CUtensorMap qm;
  if (!make_tmap_2d(&qm, Q, uint64_t(a.Lq) * a.H, D, HP)) return false;
  using C = Cfg<HP, kProducerWarps>;
  auto kern = sparse_attn_tc_kernel<HP, kProducerWarps>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) != cudaSuccess)
    return false;
  const int64_t items = int64_t(a.Lq) * a.items_per_query;
  const int grid = int(items < num_sms() ? items : num_sms());
  launch_kernel(pdl, kern, grid, 32 * C::NWARPS, C::SMEM, s, qm, static_cast<const uint16_t*>(K),
                static_cast<const uint16_t*>(V), a);
  return true;
}

bool launch_args(const void* Q, const void* K, const void* V, const AttnArgs& a, cudaStream_t s, bool pdl) {
  count_launches(1);
  if (a.H <= 16) return launch_hp<16>(Q, K, V, a, s, pdl);
  if (a.H <= 32) return launch_hp<32>(Q, K, V, a, s, pdl);
  return launch_hp<64>(Q, K, V, a, s, pdl);
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
  AttnArgs a{};
  a.idx = idx; a.Lq = int(Lq); a.Lk = int(Lk); a.k = k; a.H = H;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.kv_stride = 0;
  a.items_per_query = 1;
  a.tiles_per_item = (k + TILE - 1) / TILE;
  a.O = static_cast<uint16_t*>(O);
  return launch_args(Q, K, V, a, s, false);
}

bool launch_sparse_attn_tc_split(int batch, const void* Q, const void* Kc, const void* Vc, const int32_t* idx,
                                 int64_t capacity, int k, int H, float scale, int parts, float* Opart,
                                 float* mpart, float* lpart, cudaStream_t s, bool pdl) {
  if (batch == 0) return true;
  AttnArgs a{};
  a.idx = idx; a.Lq = batch; a.Lk = int(capacity); a.k = k; a.H = H;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.kv_stride = capacity;
  a.items_per_query = parts;
  a.tiles_per_item = ((k + TILE - 1) / TILE + parts - 1) / parts;
  a.O = nullptr;
  a.Opart = Opart; a.mpart = mpart; a.lpart = lpart;
  return launch_args(Q, Kc, Vc, a, s, pdl);
}

// Host side: whether a bounded wait of this kernel gave up on the current
// device since the flag was last cleared (synchronous copy; -1 on a CUDA error).
int attn_wait_flag(bool reset) {
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_attn_err, sizeof v) != cudaSuccess) return -1;
  if (reset && v) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_attn_err, &zero, sizeof zero) != cudaSuccess) return -1;
  }
  return v != 0;
}

}  // namespace hsa
