// Sparse softmax attention on tcgen05 tensor cores (sm_100a), multi-query:
// all H heads of a query share its k kept keys (the HISA page's "drop-in
// replacement" paragraph: the downstream sparse attention is unchanged;
// softmax(Q K^T / sqrt(d)) V as in the HiLS page's Step 4).
//
// Orientation: the kept keys, not the heads, are the MMA's M dimension, so
// every UMMA is a full 128-row tile whatever H is:
//   S^T[key][h] = Ktile[key][:] . Q[h][:]        (A = gathered K rows, K-major;
//                                                  B = the query's heads, K-major)
//   O^T[c][h]  += Vtile[key][c] . P^T[key][h]     (A = gathered V rows read
//                                                  MN-major; B = P^T, MN-major)
// A launch covers up to 64 heads (HP = 16, 32 or 64 MMA columns); more heads
// take one launch per group of 64. Head dimension d = 128, or d = 64 with the
// upper 64 rows of V^T read from a zero tile (O^T rows 64..127 stay 0).
//
// Per CTA (persistent over queries) the warp roles form a pipeline:
//   warps 0..3   producers: cp.async gathers of the kept K and V rows of each
//                128-key tile straight into the 128B-swizzled layout UMMA
//                reads (lane l loads the index of row 32w+l once per tile and
//                the copying lanes take it by shuffle); warp 0 also copies
//                each query's rows of Q (rows past its heads zero-filled);
//   warp 4       S issuer: S^T of tile g;
//   warp 5       PV issuer: O^T of tile g, so a barrier probe queued behind
//                one kind of MMA never holds up the other;
//   warps 6..21  four softmax warpgroups, warpgroup w owning heads
//                [w*HP/4, (w+1)*HP/4): thread = TMEM lane = key row of the tile.
// Softmax runs in the exp2 domain, in two passes (two launches) for a
// prefill call. The first keeps each head's running maximum from the item's
// first tile (the only cross-thread max reduction) and takes every later tile
// against it; an item whose weights then grow past 2^24 (a partial row sum
// above it, or not a number), or whose first tile left a head without a
// finite maximum, is flagged and not written. The second pass takes the
// flagged items again with a per-tile check, one hardware barrier reduction,
// that raises the maximum (and rescales O^T, l) when a tile exceeds it by more
// than 2^8; it exits at once when nothing was flagged. The decode step, whose
// parts are a few tiles long, runs the second pass alone over every part.
// P is rounded to bf16 for the second MMA; accumulation is fp32; O is
// normalised by one reciprocal of the row sum per head.
//
// A barrier probe in an MMA-issuing thread costs about as much as an MMA when
// MMAs are queued, so with two stages each issuer waits on one barrier per
// MMA group: "K tile landed and S buffer read" before S, "P written and V
// tile landed" before PV, each counting the arrivals of both producers.
//
// Every mbarrier wait is bounded. Within a softmax warpgroup all four warps
// take the same sequence of named barriers: a failed wait is folded into the
// next barrier reduction, after which the whole warpgroup leaves together.
#include <atomic>

#include "kernels.cuh"
#include "tc.cuh"

namespace hsa {

__device__ int g_attn_err;     // set when a bounded wait gives up
__device__ int g_attn_inject;  // test hook: short waits and one lost arrival

// Flagged-item lists of the prefill launches: a ring of slots, one per head
// group of a call (a slot is reused kRedoSlots groups later), each a count and
// up to kRedoSlotCap items.
constexpr int kRedoSlots = 64, kRedoSlotCap = 4096;
__device__ int g_attn_redo[kRedoSlots * (1 + kRedoSlotCap)];

namespace {

using namespace tc;

constexpr int TILE = 128;    // kept keys per MMA tile (the M dimension)
constexpr int NWG = 4;       // softmax warpgroups
constexpr int NPW = 4;       // producer warps: one kept-index row per lane
constexpr float kRescaleThreshold = 8.0f;  // log2 units (second pass)
constexpr float kFlagSum = 16777216.0f;    // 2^24: a larger partial row sum flags the item
constexpr long long kInjectWaitCycles = 1ll << 21;  // about a millisecond

template <int HP, int DH>
struct Cfg {
  static constexpr int NS = HP <= 32 ? 3 : 2;       // K/V pipeline stages
  static constexpr int HH = HP / NWG;               // heads per softmax warpgroup
  static constexpr int NSW = 4 * NWG;               // softmax warps
  static constexpr int NWARPS = NPW + 2 + NSW;      // + S issuer + PV issuer
  static constexpr int KV_BYTES = TILE * DH * 2;    // one K or V tile
  static constexpr int Q_BYTES = HP * DH * 2;       // one query's heads
  static constexpr int P_ROW = HP * 2;              // bytes of one P^T row (<= 128)
  static constexpr int P_BYTES = TILE * P_ROW;
  static constexpr int Z_BYTES = DH == 64 ? TILE * 128 : 0;  // zero upper half of V^T
  static constexpr int CPR = DH / 8;                // 16-byte chunks per K/V/Q row
  static constexpr int RPI = 32 / CPR;              // rows per warp-wide copy
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + NS * KV_BYTES;
  static constexpr int OFF_Q = OFF_V + NS * KV_BYTES;
  static constexpr int OFF_P = OFF_Q + 2 * Q_BYTES;
  static constexpr int OFF_Z = OFF_P + 2 * P_BYTES;
  static constexpr int SMEM = OFF_Z + Z_BYTES + 1024;  // + alignment slack
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
// The launch covers heads [h0, h0 + nh) of the H heads of each Q / O row.
// Each query is cut into items_per_query parts of tiles_per_item 128-key
// tiles; with one part per query the kernel writes normalised O, otherwise
// every part w = q * items_per_query + s writes its unnormalised O^T, running
// maximum and row sum for a later combination. redo[0] counts the items the
// first pass flagged, listed in redo[1 .. redo_cap] (an item once per softmax
// warpgroup that flagged it); the second pass takes them in that order, or
// every item when the count is above redo_cap or there is no list (a launch
// of the second pass alone, as the decode step makes).
struct AttnArgs {
  const uint16_t* Q;
  const int32_t* idx;
  int Lq, Lk, k, H, h0, nh;
  float scale_log2;
  int64_t kv_stride;
  int items_per_query, tiles_per_item;
  uint16_t* O;
  float *Opart, *mpart, *lpart;  // [items][H][d], [items][H], [items][H]
  int* redo;                     // [1 + redo_cap]
  int redo_cap;
};

namespace {

// Bounded wait that also gives up as soon as another role has reported a
// failure, so one lost arrival cannot keep any warp spinning for long.
HSA_DEV bool wait_bar(uint64_t* bar, uint32_t parity, bool& dead) {
  if (dead) return false;
  if (mbar_try_wait(bar, parity)) return true;
  // the limit is read only on this slow path: the test hook shortens it
  const long long lim = *(volatile int*)&g_attn_inject ? kInjectWaitCycles : kWaitCycles;
  if (mbar_wait_bounded(bar, parity, &g_attn_err, lim)) return true;
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

// x0,x1 = fma(x0,x1 ; s,s ; c0,c1) as one packed f32x2 instruction (round to nearest)
HSA_DEV void ffma2(float& x0, float& x1, float s, float c0, float c1) {
  asm("{\n .reg .b64 ra, rb, rc;\n mov.b64 ra, {%0, %1};\n mov.b64 rb, {%2, %2};\n"
      " mov.b64 rc, {%3, %4};\n fma.rn.f32x2 ra, ra, rb, rc;\n mov.b64 {%0, %1}, ra;\n}"
      : "+f"(x0), "+f"(x1) : "f"(s), "f"(c0), "f"(c1));
}
// a0,a1 += b0,b1 as one packed f32x2 instruction (round to nearest)
HSA_DEV void fadd2(float& a0, float& a1, float b0, float b1) {
  asm("{\n .reg .b64 ra, rb;\n mov.b64 ra, {%0, %1};\n mov.b64 rb, {%2, %3};\n"
      " add.rn.f32x2 ra, ra, rb;\n mov.b64 {%0, %1}, ra;\n}"
      : "+f"(a0), "+f"(a1) : "f"(b0), "f"(b1));
}
HSA_DEV float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
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

// Tiles of a query (or part) given where its kept list ends: the last valid
// index position is found from the last 128 entries, fetched one query ahead
// by the caller, or by a backwards search in the rare row whose tail is all
// padding. Warp-collective; every lane returns the same count.
struct TailScan {
  bool vec;
  int s0;
  HSA_DEV int4 window(const int32_t* idx, int q, int k) const {
    return vec ? __ldg(reinterpret_cast<const int4*>(idx + int64_t(q) * k + s0) + (threadIdx.x & 31))
               : make_int4(-1, -1, -1, -1);
  }
  HSA_DEV int last_valid(int4 win, const int32_t* row, int k, int Lk) const {
    const int lane = threadIdx.x & 31;
    int last = -1;
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
    return last;
  }
};

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

// VOTE false: the first pass over every item; true: the second pass over
// the flagged ones (launched in stream order after the first).
template <int HP, int DH, bool VOTE>
__global__ void __launch_bounds__(32 * Cfg<HP, DH>::NWARPS, 1) sparse_attn_tc_kernel(
    const uint16_t* __restrict__ K, const uint16_t* __restrict__ V, const AttnArgs a) {
  using C = Cfg<HP, DH>;
  const int32_t* __restrict__ idx = a.idx;
  const int Lk = a.Lk, k = a.k, H = a.H;
  const float scale_log2 = a.scale_log2;
  const int ipq = a.items_per_query, tpi = a.tiles_per_item;
  if (VOTE) griddep_wait();  // the first pass has finished its list
  const int flagged_n = VOTE && a.redo ? *a.redo : 0;
  const bool listed = VOTE && a.redo && flagged_n <= a.redo_cap;  // else every item
  const int n_items = listed ? flagged_n : a.Lq * ipq;
  if (VOTE && a.redo && flagged_n == 0) return;  // nothing flagged (the whole CTA leaves)
  // the w-th item of this pass
  auto item = [&](int w) { return listed ? a.redo[1 + w] : w; };
  constexpr int HH = C::HH;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) Bars bars;
  __shared__ uint32_t tmem_base;
  __shared__ int qinfo[2][2];  // per Q buffer: first tile, tile count
  __shared__ float red[4][HP];
  __shared__ float mh[HP];
  __shared__ float lsum[HP];
  __shared__ float linv[HP];  // 1 / lsum (0 where lsum is 0)

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nh = a.nh;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(&bars.kfull[s], NPW * 32); mbar_init(&bars.kempty[s], 1);
      mbar_init(&bars.vfull[s], NPW * 32); mbar_init(&bars.vempty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars.qfull[b], 32 + 1); mbar_init(&bars.qempty[b], 2 + C::NSW);
      mbar_init(&bars.sfull[b], 1); mbar_init(&bars.sempty[b], C::NSW);
      mbar_init(&bars.pfull[b], C::NSW); mbar_init(&bars.pempty[b], 1);
      mbar_init(&bars.sgo[b], NPW * 32 + C::NSW); mbar_init(&bars.pgo[b], NPW * 32 + C::NSW);
      // each S buffer starts out read: credit the softmax arrivals of its first use
      for (int u = 0; u < C::NSW; ++u) mbar_arrive(&bars.sgo[b]);
      mbar_init(&bars.ofull[b], 1); mbar_init(&bars.oempty[b], C::NSW);
    }
    mbar_init(&bars.done, 2);
    fence_barrier_init();
  }
  if constexpr (C::Z_BYTES > 0) {
    for (int e = threadIdx.x; e < C::Z_BYTES / 16; e += 32 * C::NWARPS)
      reinterpret_cast<uint4*>(sm + C::OFF_Z)[e] = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();  // written here, read by the MMA
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
    static_assert(TILE == 32 * NPW, "one kept-index row per producer lane");
    // the copy of (row 32 * warp + RPI * u + rsub, chunk cpk) takes the row's
    // index from lane RPI * u + rsub
    const int rsub = lane / C::CPR, cpk = lane % C::CPR;
    // shared-memory offset of (row 32 * warp + rsub, chunk cpk) in the
    // 128B-swizzled K-major tile, before the swizzle of the chunk
    const uint32_t dbase = (cpk >> 3) * (TILE * 128) + (32 * warp + rsub) * 128;
    const TailScan ts{(k & 3) == 0 && k >= 128, ((k & 3) == 0 && k >= 128) ? k - 128 : 0};
    int4 pre = int(blockIdx.x) < n_items ? ts.window(idx, item(blockIdx.x) / ipq, k) : make_int4(-1, -1, -1, -1);
    const bool inject = *(volatile int*)&g_attn_inject != 0;
    uint32_t g = 0, qn = 0;
    for (int wi = blockIdx.x; wi < n_items && !dead; wi += gridDim.x, ++qn) {
      const int w = item(wi), q = w / ipq, part = w - q * ipq;
      const int32_t* row = idx + int64_t(q) * k;
      const uint4* Kq = reinterpret_cast<const uint4*>(K + int64_t(q) * a.kv_stride * DH);
      const uint4* Vq = reinterpret_cast<const uint4*>(V + int64_t(q) * a.kv_stride * DH);
      const int4 win = pre;
      if (wi + int(gridDim.x) < n_items) pre = ts.window(idx, item(wi + gridDim.x) / ipq, k);
      const int last = ts.last_valid(win, row, k, Lk);
      const int t0 = part * tpi;                                  // this item's tiles
      const int nt = max(0, min((last + TILE) / TILE, t0 + tpi) - t0);
      const int qb = qn & 1;
      // warp 0: this query's HP head rows of Q (rows past its nh heads: zeros)
      // and its tile count; the other producers go straight on to its tiles
      if (warp == 0) {
        if (!wait_warp(&bars.qempty[qb], ((qn >> 1) & 1) ^ 1, dead)) break;
        if (lane == 0) {
          qinfo[qb][0] = t0;
          qinfo[qb][1] = nt;
          mbar_arrive(&bars.qfull[qb]);  // releases qinfo
        }
        const uint32_t qt = smem_u32(sm + C::OFF_Q + qb * C::Q_BYTES);
        const uint4* qsrc = reinterpret_cast<const uint4*>(a.Q) + (int64_t(q) * H + a.h0) * C::CPR;
        for (int e = lane; e < HP * C::CPR; e += 32) {
          const int h = e / C::CPR, c = e % C::CPR;
          const bool live = h < nh;
          cp_async16_zfill(qt + (c >> 3) * (HP * 128) + swz_offset(h, c & 7, 128),
                           live ? qsrc + h * C::CPR + c : qsrc, live);
        }
        cp_async_arrive(&bars.qfull[qb]);
      }
      for (int i = 0; i < nt && !dead; ++i, ++g) {
        const int s = g % C::NS;
        const uint32_t ph = (g / C::NS) & 1;
        // lane l fetches the kept index of row 32 * warp + l
        const int pos = (t0 + i) * TILE + 32 * warp + lane;
        const int jv = pos < k ? __ldg(row + pos) : -1;
        const int jc = ((jv >= 0 && jv < Lk) ? jv : 0) * C::CPR;  // row start, 16-byte units
        // with two stages, a K stage is free once S of the tile two back is
        // done (sfull), a V stage once its PV is done (pempty)
        if (!wait_warp(C::NS == 2 ? &bars.sfull[s] : &bars.kempty[s], ph ^ 1, dead)) break;
        const uint32_t kt = smem_u32(sm + C::OFF_K + s * C::KV_BYTES) + dbase;
        int jr[32 / C::RPI];
#pragma unroll
        for (int u = 0; u < 32 / C::RPI; ++u) {
          const int rr = C::RPI * u + rsub;
          jr[u] = __shfl_sync(kFull, jc, rr) + cpk;
          cp_async16(kt + u * (C::RPI * 128) + ((uint32_t((cpk & 7) ^ (rr & 7))) << 4), Kq + jr[u]);
        }
        // test hook: one producer's K arrival on the first tile of CTA 0 is lost
        if (!(inject && blockIdx.x == 0 && g == 0 && warp == 0 && lane == 0))
          cp_async_arrive(C::NS == 2 ? &bars.sgo[s] : &bars.kfull[s]);
        if (!wait_warp(C::NS == 2 ? &bars.pempty[s] : &bars.vempty[s], ph ^ 1, dead)) break;
        const uint32_t vt = smem_u32(sm + C::OFF_V + s * C::KV_BYTES) + dbase;
#pragma unroll
        for (int u = 0; u < 32 / C::RPI; ++u)
          cp_async16(vt + u * (C::RPI * 128) + ((uint32_t((cpk & 7) ^ ((C::RPI * u + rsub) & 7))) << 4), Vq + jr[u]);
        cp_async_arrive(C::NS == 2 ? &bars.pgo[s] : &bars.vfull[s]);
      }
    }
    cp_async_wait_all();  // every copy has landed before the CTA may exit
  } else if (warp == NPW) {
    // ------------------------------------------------------------ S issuer
    if (lane == 0) {
      constexpr uint32_t id_s = idesc_bf16(128, HP, false, false);
      uint32_t g = 0, qn = 0;
      for (int wi = blockIdx.x; wi < n_items && !dead; wi += gridDim.x, ++qn) {
        const int qb = qn & 1;
        if (!wait_bar(&bars.qfull[qb], (qn >> 1) & 1, dead)) break;
        const int nt = qinfo[qb][1];
        if (nt == 0) { mbar_arrive(&bars.qempty[qb]); continue; }
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
          for (int ks = 0; ks < DH / 16; ++ks)
            mma_bf16_split(tmem + sb * HP, klo + (((ks / 4) * TILE * 128 + (ks % 4) * 32) >> 4), khi,
                           qlo + (((ks / 4) * HP * 128 + (ks % 4) * 32) >> 4), qhi, id_s, ks > 0 ? 1u : 0u);
          if (C::NS != 2) mma_commit(&bars.kempty[s]);
          mma_commit(&bars.sfull[sb]);
          if (i == nt - 1) mma_commit(&bars.qempty[qb]);
        }
      }
      mma_commit(&bars.done);  // counts once, when this thread's MMAs are complete
      bool d2 = false;
      wait_bar(&bars.done, 0, d2);
    }
    __syncwarp();
  } else if (warp == NPW + 1) {
    // ------------------------------------------------------------ PV issuer
    if (lane == 0) {
      constexpr uint32_t id_o = idesc_bf16(128, HP, true, true);
      uint32_t g = 0, qn = 0, oq = 0;
      for (int wi = blockIdx.x; wi < n_items && !dead; wi += gridDim.x, ++qn) {
        const int qb = qn & 1;
        if (!wait_bar(&bars.qfull[qb], (qn >> 1) & 1, dead)) break;
        const int nt = qinfo[qb][1];
        mbar_arrive(&bars.qempty[qb]);  // the tile count is all this thread reads of the query
        if (nt == 0) continue;
        const uint32_t ob = oq & 1;
        for (int i = 0; i < nt && !dead; ++i, ++g) {
          const int pb = g & 1, s = g % C::NS;
          if constexpr (C::NS == 2) {
            // one wait per tile: P written and V landed
            if (!wait_bar(&bars.pgo[pb], (g >> 1) & 1, dead)) break;
          } else {
            if (!wait_bar(&bars.pfull[pb], (g >> 1) & 1, dead)) break;
            if (!wait_bar(&bars.vfull[s], (g / C::NS) & 1, dead)) break;
          }
          if (i == 0 && !wait_bar(&bars.oempty[ob], ((oq >> 1) & 1) ^ 1, dead)) break;
          // the V rows landed by cp.async (generic proxy) are read by the MMA
          // (async proxy): order them across proxies after the acquire above
          fence_proxy_async_smem();
          tc_fence_after();
          const uint32_t vs = smem_u32(sm + C::OFF_V + s * C::KV_BYTES);
          // the second 64 rows of V^T: the tile's upper half, or the zero tile when d = 64
          const uint32_t lbo = DH == 128 ? TILE * 128 : smem_u32(sm + C::OFF_Z) - vs;
          const uint64_t a0 = smem_desc(vs, lbo, 1024, kSw128);
          const uint64_t b0 = smem_desc(smem_u32(sm + C::OFF_P + pb * C::P_BYTES), 16384, 8 * C::P_ROW, C::P_SWZ);
          const uint32_t d = tmem + 2 * HP + ob * HP;
          const uint32_t alo = uint32_t(a0), ahi = uint32_t(a0 >> 32), blo = uint32_t(b0), bhi = uint32_t(b0 >> 32);
#pragma unroll
          for (int ks = 0; ks < TILE / 16; ++ks)
            mma_bf16_split(d, alo + ((ks * 2048) >> 4), ahi, blo + ((ks * 16 * C::P_ROW) >> 4), bhi, id_o,
                           (i == 0 && ks == 0) ? 0u : 1u);
          if (C::NS != 2) mma_commit(&bars.vempty[s]);
          mma_commit(&bars.pempty[pb]);
          if (i == nt - 1) mma_commit(&bars.ofull[ob]);
        }
        ++oq;
      }
      mma_commit(&bars.done);
      bool d2 = false;
      wait_bar(&bars.done, 0, d2);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax / epilogue
    const int sw = warp - NPW - 2, wg = sw >> 2;
    const int bar_id = 1 + wg;
    const int quad = warp & 3;              // TMEM lane quadrant this warp may access
    const int wq = quad;                    // slot of this warp in the warpgroup's scratch rows
    const int r = quad * 32 + lane;         // key row of the tile / dim row of O^T
    const int h0 = wg * HH;                 // first head of this warpgroup
    const uint32_t lane_addr = uint32_t(quad * 32) << 16;
    uint32_t g = 0, qn = 0, oq = 0;
    for (int wi = blockIdx.x; wi < n_items; wi += gridDim.x, ++qn) {
      const int w = item(wi), q = w / ipq;
      const int qb = qn & 1;
      const bool okq = wait_all(&bars.qfull[qb], (qn >> 1) & 1, dead);
      if (wg_or(bar_id, !okq || dead)) { dead = true; break; }
      const int t0 = qinfo[qb][0], nt = qinfo[qb][1];
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.qempty[qb]);
      // this query's rows of O (head a.h0 + h0 + h of the launch's heads)
      uint16_t* orow = a.O ? a.O + (int64_t(q) * H + a.h0) * DH : nullptr;
      if (nt == 0) {
        if (orow) {
#pragma unroll
          for (int h = 0; h < HH; ++h)
            if (h0 + h < nh && r < DH) orow[(h0 + h) * DH + r] = 0;
        } else if (r < HH && h0 + r < nh) {  // an empty part: no weight in the combination
          a.mpart[int64_t(w) * H + a.h0 + h0 + r] = -INFINITY;
          a.lpart[int64_t(w) * H + a.h0 + h0 + r] = 0.f;
        }
        continue;
      }
      const uint32_t ob = oq & 1;
      const int32_t* irow = idx + int64_t(q) * k;
      // m: running maximum per head (log2 units), or 0 while the head has
      // seen no valid key (its scores so far are all -inf, so 2^(x - 0) = 0);
      // `complete`: every real head of this warpgroup has a finite maximum.
      float lp[HH], nm[HH];  // nm: the running maximum, negated
#pragma unroll
      for (int h = 0; h < HH; ++h) { lp[h] = 0.f; nm[h] = 0.f; }
      bool complete = false;
      bool quit = false;
      // (up to 32 heads: the kept index of the next tile is fetched a tile
      // ahead; with 64 heads the extra register costs more than it hides)
      constexpr bool kIdxAhead = HP <= 32;
      int j_next = kIdxAhead && t0 * TILE + r < k ? __ldg(irow + t0 * TILE + r) : -1;
      for (int i = 0; i < nt; ++i, ++g) {
        const int sb = g & 1;
        int j;
        if constexpr (kIdxAhead) {
          j = j_next;
          const int pn = (t0 + i + 1) * TILE + r;
          if (i + 1 < nt) j_next = pn < k ? __ldg(irow + pn) : -1;
        } else {
          const int pos = (t0 + i) * TILE + r;
          j = pos < k ? __ldg(irow + pos) : -1;
        }
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
        for (int h = 0; h < HH; h += 2) {
          ffma2(x[h], x[h + 1], scale_log2, nm[h], nm[h + 1]);
          tmax = fmax3(tmax, x[h], x[h + 1]);
        }
        if (!live || h0 + HH > nh) {
          tmax = -INFINITY;
#pragma unroll
          for (int h = 0; h < HH; ++h) {
            if (!live || h0 + h >= nh) x[h] = -INFINITY;
            tmax = fmaxf(tmax, x[h]);
          }
        }
        const bool mine = tmax > kRescaleThreshold || !complete;
        dead = dead || !oks;
        // (a query's first tile always sets the maxima: no vote needed; the
        // first pass takes no vote at all)
        if (i == 0 || (VOTE && wg_or(bar_id, mine || dead))) {
          if (wg_or(bar_id, dead)) { quit = true; break; }
          // raise the running maxima of this warpgroup's heads to cover the tile
#pragma unroll
          for (int h = 0; h < HH; ++h) {
            const float wm = redux_max(x[h] - nm[h]);  // the tile's scaled scores
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
            x[h] -= nm[h] + mn;  // re-centre the exponents on the new maximum
            nm[h] = -mn;
            all = all && (n != -INFINITY || h0 + h >= nh);
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
          // red[0] holds the old maxima until everyone has read them (a first
          // tile reads none: it rescales nothing)
          if (i > 0) wg_sync(bar_id);
        }
        // probabilities, partial row sums, this warpgroup's part of the P^T row
        const int pb = g & 1;
        const bool okw = wait_all(&bars.pempty[pb], ((g >> 1) & 1) ^ 1, dead);
        dead = dead || !okw;
        uint32_t w[(HH + 1) / 2];
#pragma unroll
        for (int e = 0; e < HH / 2; ++e) {
          const float p0 = ex2(x[2 * e]), p1 = ex2(x[2 * e + 1]);
          fadd2(lp[2 * e], lp[2 * e + 1], p0, p1);
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
      // first pass: a head left without a finite maximum by the first tile,
      // or a partial row sum above 2^24 (or not a number), flags the item, so
      // every p of an item not flagged is below 2^24 (the sums hold them
      // whole); the barrier also publishes the row sums
      bool flag = r < HH && h0 + r < nh && mh[h0 + r] == -INFINITY;
#pragma unroll
      for (int e = 0; e < NL; ++e) flag = flag || !(lp[e] <= kFlagSum);
      const bool flagged = wg_or(bar_id, !VOTE && flag);
      if (flagged && r == 0) {
        const int at = atomicAdd(a.redo, 1);
        if (at < a.redo_cap) a.redo[1 + at] = w;
      }
      if (r < HH) {
        const float l = red[0][h0 + r] + red[1][h0 + r] + red[2][h0 + r] + red[3][h0 + r];
        lsum[h0 + r] = l;
        linv[h0 + r] = l > 0.f ? 1.f / l : 0.f;
      }
      wg_sync(bar_id);
      const bool oko = wait_all(&bars.ofull[ob], (oq >> 1) & 1, dead);
      if (oko && !flagged) {
        tc_fence_after();
        float ov[HH];
        tmem_ld_cols<HH>(tmem + lane_addr + 2 * HP + ob * HP + h0, ov);
        if (orow) {
#pragma unroll
          for (int h = 0; h < HH; ++h) {
            if (h0 + h < nh && r < DH) orow[(h0 + h) * DH + r] = uint16_t(f32_to_bf16_rn(ov[h] * linv[h0 + h]));
          }
        } else {
          // one part of a split query: unnormalised O^T, running maximum, row sum
          float* op = a.Opart + (int64_t(w) * H + a.h0) * DH;
#pragma unroll
          for (int h = 0; h < HH; ++h)
            if (h0 + h < nh && r < DH) op[(h0 + h) * DH + r] = ov[h];
          if (r < HH && h0 + r < nh) {
            a.mpart[int64_t(w) * H + a.h0 + h0 + r] = mh[h0 + r];
            a.lpart[int64_t(w) * H + a.h0 + h0 + r] = lsum[h0 + r];
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

// 4 producer warps + 2 MMA-issuing warps + 16 softmax warps = 22 warps (80
// registers per thread).
// two_pass: the first pass and then the second over the flagged items;
// otherwise the second pass alone over every item.
template <int HP, int DH>
bool launch_hp(const AttnArgs& a, const void* K, const void* V, cudaStream_t s, bool pdl, bool two_pass) {
  using C = Cfg<HP, DH>;
  auto first = sparse_attn_tc_kernel<HP, DH, false>;
  auto second = sparse_attn_tc_kernel<HP, DH, true>;
  if (cudaFuncSetAttribute(first, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) != cudaSuccess ||
      cudaFuncSetAttribute(second, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) != cudaSuccess)
    return false;
  const int64_t items = int64_t(a.Lq) * a.items_per_query;
  const int grid = int(items < num_sms() ? items : num_sms());
  const auto Kp = static_cast<const uint16_t*>(K);
  const auto Vp = static_cast<const uint16_t*>(V);
  if (!two_pass) {
    launch_kernel(pdl, second, grid, 32 * C::NWARPS, C::SMEM, s, Kp, Vp, a);
    return true;
  }
  launch_kernel(pdl, first, grid, 32 * C::NWARPS, C::SMEM, s, Kp, Vp, a);
  // the flagged items again (its CTAs leave at once when there are none)
  launch_kernel(true, second, grid, 32 * C::NWARPS, C::SMEM, s, Kp, Vp, a);
  return true;
}

template <int DH>
bool launch_group(const AttnArgs& a, const void* K, const void* V, cudaStream_t s, bool pdl, bool two_pass) {
  if (a.nh <= 16) return launch_hp<16, DH>(a, K, V, s, pdl, two_pass);
  if (a.nh <= 32) return launch_hp<32, DH>(a, K, V, s, pdl, two_pass);
  return launch_hp<64, DH>(a, K, V, s, pdl, two_pass);
}

// Per group of up to 64 heads: with two_pass, both passes, the group taking
// the next slot of the ring for its list (count zeroed first); otherwise the
// second pass alone over every item (one launch).
bool launch_args(AttnArgs a, int d, const void* K, const void* V, cudaStream_t s, bool pdl, bool two_pass) {
  static std::atomic<unsigned> next_slot{0};
  int* ring = nullptr;
  if (two_pass && cudaGetSymbolAddress(reinterpret_cast<void**>(&ring), g_attn_redo) != cudaSuccess)
    return false;
  for (int h0 = 0; h0 < a.H; h0 += 64) {
    a.h0 = h0;
    a.nh = a.H - h0 < 64 ? a.H - h0 : 64;
    a.redo = nullptr;
    if (two_pass) {
      a.redo = ring + (next_slot.fetch_add(1) % kRedoSlots) * (1 + kRedoSlotCap);
      a.redo_cap = kRedoSlotCap;
      if (cudaMemsetAsync(a.redo, 0, sizeof(int), s) != cudaSuccess) return false;
    }
    count_launches(two_pass ? 2 : 1);
    const bool ok = d == 128 ? launch_group<128>(a, K, V, s, pdl, two_pass)
                             : launch_group<64>(a, K, V, s, pdl, two_pass);
    if (!ok) return false;
  }
  return true;
}

}  // namespace

bool tc_attn_supported(int H, int d, int64_t Lq, int64_t Lk) {
  return (d == 128 || d == 64) && H >= 1 && Lq * H < (int64_t(1) << 31) && Lk < (int64_t(1) << 31);
}

bool launch_sparse_attn_tc(int64_t Lq, const void* Q, const void* K, const void* V, const int32_t* idx,
                           int64_t Lk, int k, int H, int d, float scale, void* O, cudaStream_t s) {
  if (Lq == 0) return true;

  AttnArgs a{};
  a.Q = static_cast<const uint16_t*>(Q);
  a.idx = idx; a.Lq = int(Lq); a.Lk = int(Lk); a.k = k; a.H = H;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.kv_stride = 0;
  a.items_per_query = 1;
  a.tiles_per_item = (k + TILE - 1) / TILE;
  a.O = static_cast<uint16_t*>(O);
  return launch_args(a, d, K, V, s, false, true);
}

bool launch_sparse_attn_tc_split(int batch, const void* Q, const void* Kc, const void* Vc, const int32_t* idx,
                                 int64_t capacity, int k, int H, int d, float scale, int parts, float* Opart,
                                 float* mpart, float* lpart, cudaStream_t s, bool pdl) {
  if (batch == 0) return true;
  AttnArgs a{};
  a.Q = static_cast<const uint16_t*>(Q);
  a.idx = idx; a.Lq = batch; a.Lk = int(capacity); a.k = k; a.H = H;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.kv_stride = capacity;
  a.items_per_query = parts;
  a.tiles_per_item = ((k + TILE - 1) / TILE + parts - 1) / parts;
  a.O = nullptr;
  a.Opart = Opart; a.mpart = mpart; a.lpart = lpart;
  // parts of at most a few tiles: the per-tile vote costs less there than a second launch
  return launch_args(a, d, Kc, Vc, s, pdl, false);
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

// Host side: turn the attention's test hook on or off on the current device.
bool attn_set_inject(bool on) {
  const int v = on ? 1 : 0;
  return cudaMemcpyToSymbol(g_attn_inject, &v, sizeof v) == cudaSuccess;
}

}  // namespace hsa
