// Flash-attention prefill forward for sm_100a.
//
// One CTA owns a "unit": one 128-row query tile for NSLOT query heads of the
// same K/V group (NSLOT = 2 for D <= 128, 1 for D = 256), so every K/V tile it
// stages in shared memory serves NSLOT heads ("ggml-org/llama.cpp PR #28507",
// Setup: GQA 8; K/V shared-memory staging reused across the query rows of a
// block).  Roles, one warp each unless noted:
//
//   producer   TMA 4-D tiled loads (128-byte swizzle, 64-column boxes): Q once,
//              then K_0, V_0, K_1, V_1, ... through an NBUF-slot mbarrier ring.
//   MMA        one thread issues tcgen05.mma: S_i = Q_i K_j^T (both operands in
//              shared memory, fp32 accumulator in TMEM), then O_i += P_i V_j
//              with P_i read from TMEM (A operand) and V_j from shared memory.
//              With two slots the issue order is S0_j, O1 += P1_{j-1} V_{j-1},
//              S1_j, O0 += P0_j V_j, so while one softmax warpgroup works the
//              tensor core runs the other slot's two GEMMs.  P_i lives inside
//              S_i's TMEM columns; the next S_i into that region is issued
//              right behind the P.V that reads it (tcgen05 MMAs of one CTA
//              execute in issue order).  With one slot (D = 256) S is double
//              buffered instead and the ring streams K_0, K_1, V_0, K_2, V_1, ...
//   softmax    one warpgroup per slot, one thread per query row (TMEM lane):
//              online softmax in fp32 with the running (max, rowsum) per row
//              ("Anbeeld/beellama.cpp PR #149", Overview: fp32 rescale and
//              (max, rowsum) metadata), scale*log2(e) folded into the single
//              FFMA in front of exp2 ("AstrAI commit log,
//              gqa_prefill_attn_mma.cuh": pre-scaled Q, here without rounding
//              Q*scale to bf16), P rounded to bf16 into TMEM, O rescaled in
//              TMEM only when the running max grew by more than 2^8.
//
// CTA pairs (D = 256 with an even group size): the two CTAs of a cluster hold
// the two query heads of a K/V group (one head slot each, S double buffered),
// each loads half of every K/V tile (keys 64r..64r+63 of K, D columns
// 128r..128r+127 of V, r = the CTA's rank) and the leader issues 2-CTA MMAs
// (tcgen05 cta_group::2, M = 256 rows over the pair) that read both halves, so
// each K/V tile crosses from L2 into shared memory once per group ("ggml-org/
// llama.cpp PR #28507", Setup: GQA 8, head size 256).  The peer's loads land
// on its own barriers and a thread of the peer forwards each completion to the
// leader; the leader's MMA completions arrive on both CTAs' barriers.
//
// Causal masking: key t is visible to row s iff t <= q_offset + s; tiles past
// the last row's diagonal are never loaded.  Every pipeline wait is bounded:
// on expiry the CTA records a timeout status, drains its own copies and MMAs,
// frees TMEM and exits.
#include <cooperative_groups.h>

#include "kernels.h"
#include "ptx.cuh"

namespace gqa {
namespace {

namespace cg = cooperative_groups;

constexpr int BM = 128;   // query rows per slot (TMEM lanes)
constexpr int BN = 128;   // keys per tile
constexpr uint32_t BOX_BYTES = 128u * 128u;  // 128 rows x 64 bf16 columns
constexpr float LN2 = 0.6931471805599453f;
// Softmax exponentials: pair e of each 64-key half (e = 0..31) goes to the
// polynomial exp2_poly2 when bit e is set, else to MUFU ex2.  Moving one
// exponential in eight to the FMA pipe relieves the MUFU unit, which
// otherwise paces the tensor cores at D = 128; more than that loads the FMA
// and issue slots past the point of gain (measured).
constexpr uint32_t kPolyPairs = 0x80808080u;

// MB: the variant reads an additive mask, staged by TMA in two 64-key halves,
// in two stages where shared memory allows (D <= 128), so that the next
// tile's mask loads while both head slots still read this one.
// DK: the Q and K head size; DV: the V and O head size (DV <= DK).
// PAIR: the CTA-pair form (one head slot per CTA, half K/V tiles per CTA).
template <int DK, int DV = DK, bool MB = false, bool PAIR = false>
struct PrefillCfg {
  static constexpr int NSLOT = (DV <= 128 && !PAIR) ? 2 : 1;
  static constexpr int KB = DK / 64;   // 64-column boxes of a Q or K tile
  static constexpr int VB = DV / 64;   // and of a V tile
  static constexpr uint32_t TILE = KB * BOX_BYTES;   // a Q slot, or a ring slot (K or V)
  // PAIR: a ring slot holds half a tile: 64 keys x DK of K (KB boxes of 64
  // rows) or 128 keys x DV/2 of V (VB/2 boxes of 128 rows)
  static constexpr uint32_t RSLOT = PAIR ? TILE / 2 : TILE;
  static constexpr int NBUF = PAIR ? 5 : (DK == 64) ? 8 : (DK == 128 ? (MB ? 3 : 4) : 2);
  static constexpr int MSTAGES = DK <= 128 ? 2 : 1;   // mask stages (with MB)
  // PAIR: one more warp, whose thread in the peer relays the P-ready and
  // O-free signals of the peer's softmax warps to the leader
  static constexpr int THREADS = 128 * NSLOT + 64 + (PAIR ? 32 : 0);
  static constexpr int WARP_PRODUCER = 4 * NSLOT;
  static constexpr int WARP_MMA = 4 * NSLOT + 1;
  static constexpr int WARP_RELAY = 4 * NSLOT + 2;
  static constexpr uint32_t OFF_Q = 0;
  static constexpr uint32_t OFF_KV = NSLOT * TILE;
  static constexpr uint32_t MASK_HALF = BM * 128u;          // 128 rows x 64 bf16 keys
  static constexpr uint32_t OFF_MASK = OFF_KV + NBUF * RSLOT;
  static constexpr uint32_t OFF_BAR = OFF_MASK + (MB ? MSTAGES * 2u * MASK_HALF : 0u);
  // q_full, q_empty, kv_full[NBUF], kv_empty[NBUF], s_full[2], p_lo[2], p_hi[2],
  // pv_done[2], o_free[2], drain; with MB mask_full[MSTAGES][2], mask_empty[MSTAGES][2]
  static constexpr int NBARS = 2 + 2 * NBUF + 10 + 1 + (MB ? 4 * MSTAGES : 0);
  static constexpr uint32_t OFF_MISC = OFF_BAR + NBARS * 8;
  static constexpr uint32_t SMEM = OFF_MISC + 16 + 1024;  // + alignment slack
  // Two S buffers (one per slot, or a double buffer for one slot), P aliased
  // at the start of its S buffer, then O per slot.
  static constexpr uint32_t TMEM_S = 0;                   // S buffer b at b*128
  static constexpr uint32_t TMEM_O = 256;                 // O_i at TMEM_O + i*DV
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr int BAR_Q = 0;
  static constexpr int BAR_QE = 1;
  __host__ __device__ static constexpr int bar_full(int b) { return 2 + b; }
  __host__ __device__ static constexpr int bar_empty(int b) { return 2 + NBUF + b; }
  __host__ __device__ static constexpr int bar_s(int i) { return 2 + 2 * NBUF + i; }
  __host__ __device__ static constexpr int bar_plo(int i) { return 4 + 2 * NBUF + i; }
  __host__ __device__ static constexpr int bar_phi(int i) { return 6 + 2 * NBUF + i; }
  __host__ __device__ static constexpr int bar_pv(int i) { return 8 + 2 * NBUF + i; }
  __host__ __device__ static constexpr int bar_ofree(int i) { return 10 + 2 * NBUF + i; }
  static constexpr int BAR_DRAIN = 12 + 2 * NBUF;
  __host__ __device__ static constexpr int bar_mfull(int st, int h) { return 13 + 2 * NBUF + 2 * st + h; }
  __host__ __device__ static constexpr int bar_mempty(int st, int h) {
    return 13 + 2 * NBUF + 2 * MSTAGES + 2 * st + h;
  }
  // shared-memory offset of half h of mask stage st
  __host__ __device__ static constexpr uint32_t off_mask(int st, int h) {
    return OFF_MASK + (uint32_t)(2 * st + h) * MASK_HALF;
  }
  static_assert(256 + NSLOT * DV <= 512, "TMEM budget");
  static_assert(SMEM <= 232448, "shared memory budget");
  static_assert(DK % 64 == 0 && DV % 64 == 0 && DV <= DK, "head dims");
  static_assert(!PAIR || (DK == DV && !MB && VB % 2 == 0), "pair form: equal head sizes, no staged mask");
};

// Wait that ignores the abort flag: used only to drain in-flight work.
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > limit_ns) break;
  }
}

// Item n of the K/V ring: returns true for a V tile, false for a K tile, and
// the tile index.  Two slots: K_0, V_0, K_1, V_1, ...  One slot (double-
// buffered S): K_0, K_1, V_0, K_2, V_1, ..., K_{n-1}, V_{n-2}, V_{n-1}.
template <int NSLOT>
__device__ __forceinline__ bool ring_item(int n, int n_tiles, int& tile) {
  if (NSLOT == 2) {
    tile = n >> 1;
    return (n & 1) != 0;
  }
  if (n == 0) { tile = 0; return false; }
  if (n == 2 * n_tiles - 1) { tile = n_tiles - 1; return true; }
  const int m = n - 1;
  if ((m & 1) == 0) { tile = (m >> 1) + 1; return false; }
  tile = m >> 1;
  return true;
}

// One unit of work: a 128-row query tile for up to NSLOT heads of one K/V group.
struct Unit {
  int b, kvh, hl0, s0;
  int t0;       // first K/V tile the unit visits (a sliding window skips the rest)
  int n_tiles;  // tiles t0 .. t0 + n_tiles - 1
};

// Unit u in longest-first order: q-tiles with the most visible keys first,
// then batch, K/V head and head slot group (heads of a group adjacent, so
// their K/V tiles are shared in L2).
template <int NSLOT>
__device__ __forceinline__ Unit unit_at(int u, const PrefillParams& p) {
  const int upk = p.units_per_kvh;
  const int units_per_qt = p.B * p.Hkv * upk;
  const int qt_rev = u / units_per_qt;
  int rem = u - qt_rev * units_per_qt;
  Unit x;
  x.b = rem / (p.Hkv * upk);
  rem -= x.b * (p.Hkv * upk);
  x.kvh = rem / upk;
  x.hl0 = (rem - x.kvh * upk) * NSLOT;
  const int qt = p.causal ? (p.n_qt - 1 - qt_rev) : qt_rev;
  x.s0 = qt * BM;
  const int kv_end = p.causal ? min(p.Skv, p.q_offset + min(x.s0 + BM, p.Sq)) : p.Skv;
  const int kv_begin = p.ext.window > 0 ? max(0, p.q_offset + x.s0 - p.ext.window + 1) : 0;
  x.t0 = kv_begin / BN;
  x.n_tiles = (kv_end + BN - 1) / BN - x.t0;
  return x;
}

// The k-th unit of this CTA, or -1 when it has none left.  Units are dealt to
// the persistent CTAs row by row in alternating direction (boustrophedon),
// which with longest-first units balances the load like greedy LPT without a
// shared counter.
__device__ __forceinline__ int unit_index(int k, int total) {
  const long long G = gridDim.x, c = blockIdx.x;
  const long long u = (long long)k * G + ((k & 1) ? (G - 1 - c) : c);
  return u < total ? (int)u : -1;
}

// The same over CTA pairs: both CTAs of a cluster of two take the same units.
__device__ __forceinline__ int unit_index_pair(int k, int total) {
  const long long G = gridDim.x >> 1, c = blockIdx.x >> 1;
  const long long u = (long long)k * G + ((k & 1) ? (G - 1 - c) : c);
  return u < total ? (int)u : -1;
}

// Kernel variants by the optional logit terms they handle (plain runs none):
//   MODE_MASKS  sliding window and sink logits (no per-element arithmetic)
//   MODE_ALIBI  ALiBi bias, with or without window and sinks
//   MODE_ALIBI_MASK  an additive mask, with or without ALiBi, window and sinks
//   MODE_CAP    softcap, with or without ALiBi, window and sinks
//   MODE_CAP_MASK  softcap with an additive mask (and any other term)
constexpr int MODE_PLAIN = 0, MODE_MASKS = 1, MODE_ALIBI = 2, MODE_CAP = 3, MODE_CAP_MASK = 4, MODE_ALIBI_MASK = 5;

// Logits in log2 units of the N keys of a half tile whose first key sits at
// distance dist0 = key - pos from the query:
//   MODE_ALIBI  s c2 + slope2 (dist0 + e)
//   MODE_CAP    cap_b tanh(s cap_a) + slope2 (dist0 + e)   (slope2 = 0: no ALiBi)
// in packed pairs.  The ALiBi bias runs as four interleaved sums that start
// exact at each half tile, so no per-element index arithmetic is needed.
// MASK: 0 no mask; 1 mask read as 16-byte vectors (all N keys inside the
// mask, row 16-byte aligned); 2 mask read one key at a time, keys at or past
// nvalid read as 0; 3 mask row staged in shared memory (msm, swizzle swz).
template <int MODE, bool BIAS, int MASK, int N>
__device__ __forceinline__ void ext_logits_run(float (&v)[N], const LogitExt& x, float c2, float slope2,
                                               int dist0, const uint16_t* mk, int nvalid,
                                               const uint8_t* msm = nullptr, int swz = 0) {
  static_assert(N % 8 == 0, "whole groups of four pairs");
  const float b0 = slope2 * (float)dist0;
  float2 bias[4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
    bias[i] = make_float2(fmaf(slope2, (float)(2 * i), b0), fmaf(slope2, (float)(2 * i + 1), b0));
  const float2 step = make_float2(8.f * slope2, 8.f * slope2);
  const float2 l2e = make_float2(1.4426950408889634f, 1.4426950408889634f);
  uint4 mw = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
  for (int e = 0; e < N; e += 2) {
    const int i = (e >> 1) & 3;
    const float2 sp = make_float2(v[e], v[e + 1]);
    float2 y;
    if constexpr (MODE == MODE_ALIBI || MODE == MODE_ALIBI_MASK) {
      y = BIAS ? ffma2(sp, make_float2(c2, c2), bias[i]) : fmul2(sp, make_float2(c2, c2));
    } else {
      const float2 u = fmul2(sp, make_float2(x.cap_a, x.cap_a));
      const float2 t = make_float2(tanh_approx(u.x), tanh_approx(u.y));
      y = BIAS ? ffma2(t, make_float2(x.cap_b, x.cap_b), bias[i]) : fmul2(t, make_float2(x.cap_b, x.cap_b));
    }
    if constexpr (MASK != 0) {
      uint32_t w;
      if constexpr (MASK == 1) {
        if ((e & 7) == 0) mw = __ldg(reinterpret_cast<const uint4*>(mk + e));
        w = i == 0 ? mw.x : i == 1 ? mw.y : i == 2 ? mw.z : mw.w;
      } else if constexpr (MASK == 3) {
        // staged in shared memory: 16-byte chunk e/8 of a 128-byte swizzled row
        if ((e & 7) == 0) mw = *reinterpret_cast<const uint4*>(msm + ((uint32_t)((e >> 3) ^ swz) << 4));
        w = i == 0 ? mw.x : i == 1 ? mw.y : i == 2 ? mw.z : mw.w;
      } else {
        const uint32_t lo = e < nvalid ? (uint32_t)__ldg(mk + e) : 0u;
        const uint32_t hi = e + 1 < nvalid ? (uint32_t)__ldg(mk + e + 1) : 0u;
        w = lo | (hi << 16);
      }
      y = ffma2(make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u)), l2e, y);
    }
    v[e] = y.x;
    v[e + 1] = y.y;
    if (BIAS && i == 3) {
#pragma unroll
      for (int k = 0; k < 4; ++k) bias[k] = fadd2(bias[k], step);
    }
  }
}

template <int MODE, bool BIAS, int N>
__device__ __forceinline__ void ext_logits_m(float (&v)[N], const LogitExt& x, float c2, float slope2, int dist0,
                                             const uint16_t* mk, int nvalid, const uint8_t* msm, int swz) {
  if (MODE == MODE_ALIBI || MODE == MODE_CAP)   // no mask in these variants
    ext_logits_run<MODE, BIAS, 0>(v, x, c2, slope2, dist0, mk, nvalid);
  else if (msm != nullptr)
    ext_logits_run<MODE, BIAS, 3>(v, x, c2, slope2, dist0, mk, nvalid, msm, swz);
  else if (mk == nullptr)
    ext_logits_run<MODE, BIAS, 0>(v, x, c2, slope2, dist0, mk, nvalid);
  else if (nvalid >= N && (reinterpret_cast<uintptr_t>(mk) & 15u) == 0)
    ext_logits_run<MODE, BIAS, 1>(v, x, c2, slope2, dist0, mk, nvalid);
  else
    ext_logits_run<MODE, BIAS, 2>(v, x, c2, slope2, dist0, mk, nvalid);
}

// Logits of a half tile.  mk: this row's mask at the half's first key (or
// nullptr), nvalid: keys of the half inside the mask.  The branches sit
// outside the unrolled loops: no path pays for another.
template <int MODE, int N>
__device__ __forceinline__ void ext_logits(float (&v)[N], const LogitExt& x, float c2, float slope2, int dist0,
                                           const uint16_t* mk, int nvalid, const uint8_t* msm = nullptr,
                                           int swz = 0) {
  if (x.alibi)
    ext_logits_m<MODE, true>(v, x, c2, slope2, dist0, mk, nvalid, msm, swz);
  else
    ext_logits_m<MODE, false>(v, x, c2, slope2, dist0, mk, nvalid, msm, swz);
}

// Columns outside [cb, cl) become -inf.
template <int N>
__device__ __forceinline__ void mask_cols(float (&v)[N], int cb, int cl) {
#pragma unroll
  for (int e = 0; e < N; ++e) v[e] = (e < cl && e >= cb) ? v[e] : -INFINITY;
}

// Row maximum: eight independent 3-input max chains, then a small tree.
template <int N>
__device__ __forceinline__ float row_max(const float (&v)[N]) {
  static_assert(N % 16 == 0, "row_max takes multiples of 16 columns");
  float mxc[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) mxc[c] = fmaxf(v[2 * c], v[2 * c + 1]);
#pragma unroll
  for (int e = 16; e < N; e += 16) {
#pragma unroll
    for (int c = 0; c < 8; ++c) mxc[c] = fmax3(mxc[c], v[e + 2 * c], v[e + 2 * c + 1]);
  }
  return fmax3(fmax3(mxc[0], mxc[1], mxc[2]), fmax3(mxc[3], mxc[4], mxc[5]), fmaxf(mxc[6], mxc[7]));
}

// PAIR: launched in clusters of two CTAs; tm_k then tiles K in 64-key boxes.
template <int DK, int DV, int MODE, bool PAIR = false>
__global__ void __launch_bounds__(PrefillCfg<DK, DV, MODE == MODE_ALIBI_MASK || MODE == MODE_CAP_MASK, PAIR>::THREADS, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_m,
                   const PrefillParams p) {
  constexpr bool MB = MODE == MODE_ALIBI_MASK || MODE == MODE_CAP_MASK;
  using C = PrefillCfg<DK, DV, MB, PAIR>;
  constexpr int D = DV;   // the output head size
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + C::OFF_MISC + 4);
  auto bar = [&](int i) -> uint32_t { return base + C::OFF_BAR + 8u * (uint32_t)i; };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int total_units = p.n_qt * p.B * p.Hkv * p.units_per_kvh;
  // PAIR: this CTA's rank in its cluster of two (0 leads: it issues the MMAs)
  // and the pair-aware unit order
  const uint32_t rank = PAIR ? (blockIdx.x & 1u) : 0u;
  constexpr int UG = PAIR ? 2 : C::NSLOT;   // query heads per unit
  auto next_unit = [&](int k) -> int { return PAIR ? unit_index_pair(k, total_units) : unit_index(k, total_units); };
  // Waits on barriers that the peer arrives on (PAIR leader) acquire at cluster scope
  auto wait_x = [&](uint32_t b, uint32_t parity, const Watchdog& w) -> bool {
    return PAIR ? mbar_wait_cluster(b, parity, w) : mbar_wait(b, parity, w);
  };
  // With ALiBi the bias grows toward each query's own position: visiting a
  // unit's K/V tiles newest first sets the running maximum on the first tile
  // and spares the O rescales (the tile order does not change the result).
  const bool rev_alibi = MODE >= MODE_ALIBI && p.ext.alibi != 0;
  // In the CTA-pair form, units a cluster takes second, fourth, ... (odd k)
  // also run newest first: they start while the first wave's most recent K/V
  // tiles are still in L2 and reach the oldest tiles last, instead of
  // re-reading those from DRAM first (prefill at depth: DRAM reads 173 -> 130
  // MB).  Every role derives a unit's tile order from the same k.
  auto unit_rev = [&](int k) -> bool { return rev_alibi || (PAIR && (k & 1) != 0); };

  if (threadIdx.x == 0) {
    // PAIR: the leader's Q and ring barriers also count the peer's forwarded
    // completion; P and O-free barriers count one arrival per softmax warp,
    // plus (leader) the relayed arrival of the peer's four (the single-CTA
    // form: one per softmax thread)
    const uint32_t nfull = (PAIR && rank == 0) ? 2u : 1u;
    const uint32_t nsoft = PAIR ? (rank == 0 ? 5u : 4u) : 128u;
    mbar_init(bar(C::BAR_Q), nfull);
    mbar_init(bar(C::BAR_QE), 1);
    for (int i = 0; i < C::NBUF; ++i) {
      mbar_init(bar(C::bar_full(i)), nfull);
      mbar_init(bar(C::bar_empty(i)), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(C::bar_s(i)), 1);
      mbar_init(bar(C::bar_plo(i)), nsoft);
      mbar_init(bar(C::bar_phi(i)), nsoft);
      mbar_init(bar(C::bar_pv(i)), 1);
      mbar_init(bar(C::bar_ofree(i)), nsoft);
    }
    mbar_init(bar(C::BAR_DRAIN), 1);
    if constexpr (MB) {
      for (int st = 0; st < C::MSTAGES; ++st)
        for (int h = 0; h < 2; ++h) {
          mbar_init(bar(C::bar_mfull(st, h)), 1);
          mbar_init(bar(C::bar_mempty(st, h)), 4 * C::NSLOT);   // one arrival per softmax warp
        }
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == C::WARP_MMA) {
    if constexpr (PAIR) {
      tmem_alloc2(smem_u32(tmem_slot), C::TMEM_COLS);
      tmem_relinquish2();
    } else {
      tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  if constexpr (PAIR) {
    // both CTAs' barriers are initialised before either arrives on the other's
    cg::this_cluster().sync();
  } else {
    __syncthreads();
  }
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const Watchdog wd{abort_flag, p.status, p.timeout_ns};

  int issued = 0;    // producer: K/V ring items issued
  int q_issued = 0;  // producer: Q tiles issued (one per unit)
  int m_issued = 0;  // producer lane 1: mask tiles issued

  if (warp == C::WARP_PRODUCER) {
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      int n = 0;
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int u = next_unit(k);
        if (u < 0) break;
        const Unit x = unit_at<UG>(u, p);
        // the previous unit's last S MMA must be done reading Q
        if (k > 0 && !mbar_wait(bar(C::BAR_QE), (uint32_t)(k - 1) & 1u, wd)) break;
        if constexpr (PAIR) {
          // this CTA's head of the pair
          mbar_arrive_expect_tx(bar(C::BAR_Q), C::TILE);
          for (int kb = 0; kb < C::KB; ++kb)
            tma_load_4d(base + C::OFF_Q + kb * BOX_BYTES, &tm_q, bar(C::BAR_Q), kb * 64,
                        x.kvh * p.g + x.hl0 + (int)rank, x.s0, x.b);
        } else {
          int nact = 0;
          for (int i = 0; i < C::NSLOT; ++i) nact += (x.hl0 + i < p.g) ? 1 : 0;
          mbar_arrive_expect_tx(bar(C::BAR_Q), (uint32_t)nact * C::TILE);
          for (int i = 0; i < C::NSLOT; ++i) {
            if (x.hl0 + i >= p.g) continue;
            const int h = x.kvh * p.g + x.hl0 + i;
            for (int kb = 0; kb < C::KB; ++kb)
              tma_load_4d(base + C::OFF_Q + i * C::TILE + kb * BOX_BYTES, &tm_q, bar(C::BAR_Q), kb * 64, h,
                          x.s0, x.b);
          }
        }
        q_issued = k + 1;
        for (int m = 0; m < 2 * x.n_tiles; ++m, ++n) {
          const int buf = n % C::NBUF;
          const int use = n / C::NBUF;
          if (use > 0 && !mbar_wait(bar(C::bar_empty(buf)), (uint32_t)(use - 1) & 1u, wd)) { ok = false; break; }
          int tile;
          const bool is_v = ring_item<C::NSLOT>(m, x.n_tiles, tile);
          const int key0 = (x.t0 + (unit_rev(k) ? x.n_tiles - 1 - tile : tile)) * BN;
          const uint32_t dst = base + C::OFF_KV + buf * C::RSLOT;
          // a K or V tile (VB boxes for V when DV < DK), or half of one (PAIR)
          mbar_arrive_expect_tx(bar(C::bar_full(buf)), PAIR ? C::RSLOT : (uint32_t)(is_v ? C::VB : C::KB) * BOX_BYTES);
          if constexpr (PAIR) {
            if (is_v) {
              // V: all 128 keys, D columns rank*DV/2 .. (rank+1)*DV/2 - 1
              for (int vb = 0; vb < C::VB / 2; ++vb)
                tma_load_4d(dst + vb * BOX_BYTES, &tm_v, bar(C::bar_full(buf)), (int)rank * (DV / 2) + vb * 64, x.kvh,
                            key0, x.b);
            } else {
              // K: keys key0 + 64*rank .. + 63 (tm_k tiles K in 64-key boxes)
              for (int kb = 0; kb < C::KB; ++kb)
                tma_load_4d(dst + kb * (BOX_BYTES / 2), &tm_k, bar(C::bar_full(buf)), kb * 64, x.kvh,
                            key0 + 64 * (int)rank, x.b);
            }
          } else {
            const CUtensorMap* tm = is_v ? &tm_v : &tm_k;
            const int nb = is_v ? C::VB : C::KB;
            for (int kb = 0; kb < nb; ++kb)
              tma_load_4d(dst + kb * BOX_BYTES, tm, bar(C::bar_full(buf)), kb * 64, x.kvh, key0, x.b);
          }
          issued = n + 1;
        }
      }
    } else if (MB && lane == 1 && p.mask_tma) {
      // The additive mask of every tile, in the K/V stream's tile order, as
      // two 64-key halves (16 KB each, 128-byte swizzled rows); a half is
      // refilled once every softmax warp has released it.  Each slot visits
      // every tile (one slot, or an even group size), so the counts agree.
      tma_prefetch_desc(&tm_m);
      bool ok = true;
      int tg = 0;   // this CTA's tiles so far
      for (int k = 0; ok; ++k) {
        const int u = next_unit(k);
        if (u < 0) break;
        const Unit x = unit_at<UG>(u, p);
        for (int j = 0; ok && j < x.n_tiles; ++j, ++tg) {
          const int key0 = (x.t0 + (unit_rev(k) ? x.n_tiles - 1 - j : j)) * BN;
          const int st = tg % C::MSTAGES, use = tg / C::MSTAGES;   // stage, and its use count
          for (int h = 0; h < 2; ++h) {
            if (use > 0 && !mbar_wait(bar(C::bar_mempty(st, h)), (uint32_t)(use - 1) & 1u, wd)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(bar(C::bar_mfull(st, h)), C::MASK_HALF);
            tma_load_4d(base + C::off_mask(st, h), &tm_m, bar(C::bar_mfull(st, h)), key0 + 64 * h, x.s0,
                        p.ext.mask_sb != 0 ? x.b : 0, 0);
          }
          m_issued = tg + 1;
        }
      }
    }
  } else if (warp == C::WARP_MMA) {
    if (PAIR && rank == 1 && lane == 0) {
      // The peer's loads complete on its own barriers; forward each completion
      // (Q of every unit, then its ring items in order) to the leader's
      // barrier of the same index, where the MMAs wait for both halves.
      int n = 0;
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int u = next_unit(k);
        if (u < 0) break;
        const Unit x = unit_at<UG>(u, p);
        if (!(ok = mbar_wait(bar(C::BAR_Q), (uint32_t)k & 1u, wd))) break;
        mbar_relay_cluster(mapa_shared(bar(C::BAR_Q), 0));
        for (int m = 0; m < 2 * x.n_tiles; ++m, ++n) {
          if (!(ok = mbar_wait(bar(C::bar_full(n % C::NBUF)), (uint32_t)(n / C::NBUF) & 1u, wd))) break;
          mbar_relay_cluster(mapa_shared(bar(C::bar_full(n % C::NBUF)), 0));
        }
      }
    } else if (lane == 0 && (!PAIR || rank == 0)) {
      // PAIR: 2-CTA MMAs over M = 256 rows (both heads of the pair)
      constexpr uint32_t IDESC_QK = idesc_bf16_f32(PAIR ? 2 * BM : BM, BN, false, false);
      constexpr uint32_t IDESC_PV = idesc_bf16_f32(PAIR ? 2 * BM : BM, D, false, true);
      // completions arrive on this CTA's barrier, or on the barrier at the same
      // offset in both CTAs of the pair
      auto commit = [&](uint32_t b) {
        if constexpr (PAIR) mma_commit_pair(b);
        else mma_commit(b);
      };
      auto wait_full = [&](int n) -> bool {
        if (!wait_x(bar(C::bar_full(n % C::NBUF)), (uint32_t)(n / C::NBUF) & 1u, wd)) return false;
        tc_fence_after();
        return true;
      };

      // Descriptors are built once; a K-step only advances the start-address
      // field (bits 0-13, in 16-byte units), which never carries for these
      // offsets since every tile lies below 256 KB of shared memory.
      const uint64_t qdesc0 = sdesc_sw128(base + C::OFF_Q, 16, 1024);
      const uint64_t kdesc0 = sdesc_sw128(base + C::OFF_KV, 16, 1024);
      const uint64_t vdesc0 = sdesc_sw128(base + C::OFF_KV, BOX_BYTES, 1024);
      // K boxes: 128 rows (64 in the pair form) of 128 bytes
      constexpr uint32_t KBOX = PAIR ? BOX_BYTES / 2 : BOX_BYTES;
      // S buffer sb = Q(qslot) K^T
      auto gemm_s = [&](int sb, int qslot, int ring_n) {
        const uint64_t qd = qdesc0 + (uint64_t)(((uint32_t)qslot * C::TILE) >> 4);
        const uint64_t kd = kdesc0 + (uint64_t)(((uint32_t)(ring_n % C::NBUF) * C::RSLOT) >> 4);
#pragma unroll
        for (int kk = 0; kk < DK / 16; ++kk) {
          const uint64_t qo = (uint64_t)((((uint32_t)(kk >> 2) * BOX_BYTES) + (uint32_t)(kk & 3) * 32u) >> 4);
          const uint64_t ko = (uint64_t)((((uint32_t)(kk >> 2) * KBOX) + (uint32_t)(kk & 3) * 32u) >> 4);
          if constexpr (PAIR)
            mma_ss_pair(tmem + C::TMEM_S + sb * 128, qd + qo, kd + ko, IDESC_QK, kk > 0 ? 1u : 0u);
          else
            mma_ss(tmem + C::TMEM_S + sb * 128, qd + qo, kd + ko, IDESC_QK, kk > 0 ? 1u : 0u);
        }
      };
      // O(oslot) (+)= P(from S buffer pb) V, each half of P as soon as it is
      // in TMEM (phase: completion index of that buffer's P barriers)
      auto gemm_pv = [&](int oslot, int pb, int ring_n, bool first, uint32_t phase) -> bool {
        const uint64_t vd = vdesc0 + (uint64_t)(((uint32_t)(ring_n % C::NBUF) * C::RSLOT) >> 4);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          if (!wait_x(bar(half == 0 ? C::bar_plo(pb) : C::bar_phi(pb)), phase & 1u, wd)) return false;
          tc_fence_after();
#pragma unroll
          for (int kk = half * (BN / 32); kk < (half + 1) * (BN / 32); ++kk) {
            if constexpr (PAIR)
              mma_ts_pair(tmem + C::TMEM_O + oslot * D, tmem + C::TMEM_S + pb * 128 + kk * 8,
                          vd + (uint64_t)((kk * 2048u) >> 4), IDESC_PV, (!first || kk > 0) ? 1u : 0u);
            else
              mma_ts(tmem + C::TMEM_O + oslot * D, tmem + C::TMEM_S + pb * 128 + kk * 8,
                     vd + (uint64_t)((kk * 2048u) >> 4), IDESC_PV, (!first || kk > 0) ? 1u : 0u);
          }
        }
        return true;
      };
      auto wait_ofree = [&](int slot, int units_done) -> bool {
        // the previous unit's epilogue on this slot must be done reading O
        if (units_done == 0) return true;
        if (!wait_x(bar(C::bar_ofree(slot)), (uint32_t)(units_done - 1) & 1u, wd)) return false;
        tc_fence_after();
        return true;
      };
      bool ok = true;
      int n = 0;                       // ring items consumed
      int T0 = 0, T1 = 0;              // tiles completed per slot (barrier phases)
      int U0 = 0, U1 = 0;              // units completed per slot
      for (int k = 0; ok; ++k) {
        const int u = next_unit(k);
        if (u < 0) break;
        const Unit x = unit_at<UG>(u, p);
        const int nt = x.n_tiles;
        const bool act1 = (C::NSLOT == 2) && (x.hl0 + 1 < p.g);
        if (!(ok = wait_x(bar(C::BAR_Q), (uint32_t)k & 1u, wd))) break;
        tc_fence_after();
        if (C::NSLOT == 2) {
          // tile 0
          if (!(ok = wait_full(n))) break;
          gemm_s(0, 0, n);
          commit(bar(C::bar_s(0)));
          if (act1) {
            gemm_s(1, 1, n);
            commit(bar(C::bar_s(1)));
          }
          if (nt == 1) commit(bar(C::BAR_QE));            // last S of the unit
          commit(bar(C::bar_empty(n % C::NBUF)));
          if (!(ok = wait_full(n + 1) && wait_ofree(0, U0) &&
                     gemm_pv(0, 0, n + 1, true, (uint32_t)T0)))
            break;
          commit(bar(C::bar_pv(0)));
          for (int i = 1; i < nt; ++i) {
            const int nk = n + 2 * i;
            if (!(ok = wait_full(nk))) break;
            gemm_s(0, 0, nk);                                 // S0_i (behind O0 += P0_{i-1} V_{i-1})
            commit(bar(C::bar_s(0)));
            if (act1) {
              if (!(ok = (i > 1 || wait_ofree(1, U1)) &&
                         gemm_pv(1, 1, nk - 1, i == 1, (uint32_t)(T1 + i - 1))))
                break;                                        // O1 += P1_{i-1} V_{i-1}
              commit(bar(C::bar_pv(1)));
            }
            commit(bar(C::bar_empty((nk - 1) % C::NBUF)));  // V_{i-1} done
            if (act1) {
              gemm_s(1, 1, nk);                               // S1_i (behind the P1 read)
              commit(bar(C::bar_s(1)));
            }
            if (i == nt - 1) commit(bar(C::BAR_QE));      // last S of the unit
            commit(bar(C::bar_empty(nk % C::NBUF)));      // K_i done
            if (!(ok = wait_full(nk + 1) && gemm_pv(0, 0, nk + 1, false, (uint32_t)(T0 + i)))) break;
            commit(bar(C::bar_pv(0)));                    // O0 += P0_i V_i
          }
          if (!ok) break;
          const int nv = n + 2 * nt - 1;
          if (act1) {
            if (!(ok = (nt > 1 || wait_ofree(1, U1)) &&
                       gemm_pv(1, 1, nv, nt == 1, (uint32_t)(T1 + nt - 1))))
              break;
            commit(bar(C::bar_pv(1)));
          }
          commit(bar(C::bar_empty(nv % C::NBUF)));
          T0 += nt;
          ++U0;
          if (act1) {
            T1 += nt;
            ++U1;
          }
        } else {
          // one slot, S double buffered across tiles and units: buffer (T0 + j) % 2
          if (!(ok = wait_full(n))) break;
          gemm_s(T0 & 1, 0, n);
          commit(bar(C::bar_s(T0 & 1)));
          if (nt == 1) commit(bar(C::BAR_QE));
          commit(bar(C::bar_empty(n % C::NBUF)));
          ++n;
          for (int j = 0; j < nt; ++j) {
            const int G = T0 + j;
            if (j + 1 < nt) {
              if (!(ok = wait_full(n))) break;
              gemm_s((G + 1) & 1, 0, n);                      // behind the P.V that read this buffer
              commit(bar(C::bar_s((G + 1) & 1)));
              if (j + 2 == nt) commit(bar(C::BAR_QE));    // last S of the unit
              commit(bar(C::bar_empty(n % C::NBUF)));
              ++n;
            }
            if (!(ok = wait_full(n) && (j > 0 || wait_ofree(0, U0)) &&
                       gemm_pv(0, G & 1, n, j == 0, (uint32_t)(G >> 1))))
              break;
            commit(bar(C::bar_pv(0)));
            commit(bar(C::bar_empty(n % C::NBUF)));
            ++n;
          }
          if (!ok) break;
          T0 += nt;
          ++U0;
          continue;
        }
        n += 2 * nt;
      }
    }
  } else if (PAIR && warp == C::WARP_RELAY) {
    if (rank == 1 && lane == 0) {
      // The peer's softmax warps arrive on its own P and O-free barriers
      // (a remote arrive stalls the arriving warp); relay each completed
      // phase, in the order the leader's MMAs wait for them, to the leader's
      // barrier of the same index.
      int T = 0;
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int u = next_unit(k);
        if (u < 0) break;
        const Unit x = unit_at<UG>(u, p);
        for (int j = 0; ok && j < x.n_tiles; ++j) {
          const int G = T + j;
          for (int half = 0; half < 2; ++half) {
            const uint32_t b = bar(half == 0 ? C::bar_plo(G & 1) : C::bar_phi(G & 1));
            if (!(ok = mbar_wait(b, (uint32_t)(G >> 1) & 1u, wd))) break;
            mbar_relay_cluster(mapa_shared(b, 0));
          }
        }
        if (!ok || !(ok = mbar_wait(bar(C::bar_ofree(0)), (uint32_t)k & 1u, wd))) break;
        mbar_relay_cluster(mapa_shared(bar(C::bar_ofree(0)), 0));
        T += x.n_tiles;
      }
    }
  } else {
    // ---- softmax warpgroups: warp w serves slot w/4, TMEM lanes 32*(w%4).. ----
    const int slot = warp >> 2;
    const int wq = warp & 3;
    const int r = wq * 32 + lane;
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const uint32_t tO = tmem + lane_off + C::TMEM_O + slot * D;
    const float c2 = p.c2;
    int T = 0;  // tiles this slot completed in earlier units (barrier phases)
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int u = next_unit(k);
      if (u < 0) break;
      const Unit x = unit_at<UG>(u, p);
      const int hl = x.hl0 + (PAIR ? (int)rank : slot);
      if (hl >= p.g) continue;  // slot unused in this unit (odd group size)
      const int n_tiles = x.n_tiles;
      const int h = x.kvh * p.g + hl;
      const int s_row = x.s0 + r;
      const int pos = p.q_offset + s_row;
      const int vis_end = p.causal ? min(p.Skv, pos + 1) : p.Skv;
      const int vis_begin = (MODE != MODE_PLAIN && p.ext.window > 0) ? pos - p.ext.window + 1 : 0;
      const float slope2 =
          (MODE >= MODE_ALIBI && p.ext.alibi) ? alibi_slope_log2e(h, p.ext.l2m0, p.ext.l2m1, p.ext.n2) : 0.f;
      // this row's mask (padding rows past Sq read the last row's: never stored)
      const uint16_t* mrow = ((MODE == MODE_ALIBI_MASK || MODE == MODE_CAP_MASK) && p.ext.mask != nullptr)
                                 ? p.ext.mask + (size_t)x.b * p.ext.mask_sb + (size_t)min(s_row, p.Sq - 1) * p.ext.mask_sr
                                 : nullptr;
      float m_use = -INFINITY, l = 0.f;
      for (int j = 0; j < n_tiles; ++j) {
        const int G = T + j;
        // S buffer and its phase: per slot, or alternating for one slot
        const int sb = (C::NSLOT == 2) ? slot : (G & 1);
        const uint32_t ph = (C::NSLOT == 2) ? ((uint32_t)G & 1u) : ((uint32_t)(G >> 1) & 1u);
        const uint32_t tS = tmem + lane_off + C::TMEM_S + sb * 128;
        // a give-up must be warp-uniform: TMEM loads/stores are warp-collective
        const bool got = mbar_wait(bar(C::bar_s(sb)), ph, wd);
        if (__any_sync(0xffffffffu, !got)) { ok = false; break; }
        tc_fence_after();
        const int key0 = (x.t0 + (unit_rev(k) ? n_tiles - 1 - j : j)) * BN;
        const int cl = vis_end - key0;    // visible columns of this tile: [cb, cl)
        const int cb = vis_begin - key0;
        const bool tile_masked = __any_sync(0xffffffffu, cl < BN || cb > 0);
        float sv[BN];
        float mx;
        if constexpr (MODE >= MODE_ALIBI) {
          // logits in log2 units with the ALiBi / softcap terms; keys 64-127
          // first, for their maximum only, so that one half of the row is
          // live at a time.  Their logits go back to their own TMEM columns
          // (P only ever covers columns 0-63), where half 1 below reads them.
          // staged mask: wait for this tile's halves (tile G of this slot,
          // and of the producer's mask stream)
          const bool mstaged = MB && p.mask_tma;
          const uint8_t* msm_hi = nullptr;
          const uint8_t* msm_lo = nullptr;
          int mst = 0;
          if (mstaged) {
            mst = G % C::MSTAGES;
            const uint32_t mph = (uint32_t)(G / C::MSTAGES) & 1u;
            const bool got_m =
                mbar_wait(bar(C::bar_mfull(mst, 1)), mph, wd) && mbar_wait(bar(C::bar_mfull(mst, 0)), mph, wd);
            if (__any_sync(0xffffffffu, !got_m)) { ok = false; break; }
            msm_lo = gbase + C::off_mask(mst, 0) + (uint32_t)r * 128u;
            msm_hi = gbase + C::off_mask(mst, 1) + (uint32_t)r * 128u;
          }
          float sh[BN / 2];
          tmem_ld64(tS + BN / 2, sh);
          ext_logits<MODE>(sh, p.ext, c2, slope2, key0 + BN / 2 - pos, mrow ? mrow + key0 + BN / 2 : nullptr,
                           p.Skv - (key0 + BN / 2), msm_hi, r & 7);
          {
            uint32_t u[BN / 2];
#pragma unroll
            for (int e = 0; e < BN / 2; ++e) u[e] = __float_as_uint(sh[e]);
            tmem_st64(tS + BN / 2, u);
          }
          if (tile_masked) mask_cols(sh, cb - BN / 2, cl - BN / 2);
          const float mx_hi = row_max(sh);
          float (&slo)[BN / 2] = *reinterpret_cast<float(*)[BN / 2]>(sv);
          tmem_ld64(tS, slo);
          ext_logits<MODE>(slo, p.ext, c2, slope2, key0 - pos, mrow ? mrow + key0 : nullptr, p.Skv - key0, msm_lo,
                           r & 7);
          if (mstaged) {
            // both halves read into registers: release them to the producer
            __syncwarp();
            if (lane == 0) {
              mbar_arrive(bar(C::bar_mempty(mst, 0)));
              mbar_arrive(bar(C::bar_mempty(mst, 1)));
            }
          }
          if (tile_masked) mask_cols(slo, cb, cl);
          mx = fmaxf(mx_hi, row_max(slo));
        } else {
          // one TMEM read of the whole 128-column S row
          tmem_ld128(tS, sv);
          if (tile_masked) mask_cols(sv, cb, cl);
          mx = row_max(sv);
        }
        const float m_tile = (MODE >= MODE_ALIBI) ? mx : mx * c2;
        float m_new = m_use, alpha = 1.f;
        if (m_tile > m_use + 8.f) {
          m_new = m_tile;
          alpha = ex2_approx(m_use - m_new);
        }
        const float m_sub = (m_new == -INFINITY) ? 0.f : m_new;
        if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
          // O must be rescaled before the first half of P is handed over.
          // Two slots: S_i(j) was issued behind O_i += P_i(j-1) V, so its
          // completion implies that P.V completed.  One slot: S(j) was issued
          // before that P.V, so wait for it here.
          if (C::NSLOT == 1) {
            const bool got_pv = mbar_wait(bar(C::bar_pv(0)), (uint32_t)(G - 1) & 1u, wd);
            if (__any_sync(0xffffffffu, !got_pv)) { ok = false; break; }
            tc_fence_after();
          }
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            float v[32];
            tmem_ld32(tO + 32 * c, v);
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] *= alpha;
            tmem_st32(tO + 32 * c, v);
          }
        }
        // p = 2^(s*c2 - m): one packed FFMA per pair, ex2 per element, packed
        // partial sums, bf16 pairs for the P.V operand (masked s = -inf -> p = 0).
        // P is handed over in two halves (keys 0-63, then 64-127) so the P.V
        // MMAs on the first half overlap the exponentials of the second.
        const float2 c2v = (MODE >= MODE_ALIBI) ? make_float2(1.f, 1.f) : make_float2(c2, c2);
        const float2 nmv = make_float2(-m_sub, -m_sub);
        float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
        // half 0: keys 0-63 from the registers; P lands on TMEM columns 0-31,
        // whose S values were read above
        {
          uint32_t pk[BN / 4];
#pragma unroll
          for (int e = 0; e < BN / 4; ++e) {
            const float2 x = ffma2(make_float2(sv[2 * e], sv[2 * e + 1]), c2v, nmv);
            const float2 pr = ((kPolyPairs >> e) & 1u) ? exp2_poly2(x)
                                                              : make_float2(ex2_approx(x.x), ex2_approx(x.y));
            if (e & 1) acc1 = fadd2(acc1, pr); else acc0 = fadd2(acc0, pr);
            pk[e] = pack_bf16x2(pr.x, pr.y);
          }
          tmem_st32u(tS, pk);
          tmem_wait_st();
          tc_fence_before();
          if constexpr (PAIR) {
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(C::bar_plo(sb)));
          } else {
            mbar_arrive(bar(C::bar_plo(sb)));
          }
        }
        // half 1: keys 64-127, re-read from TMEM columns 64-127 (P only ever
        // covers columns 0-63), so their registers need not stay live above
        {
          float sh[BN / 2];
          tmem_ld64(tS + BN / 2, sh);   // with ALiBi / softcap: logits stored above
          if (tile_masked) mask_cols(sh, cb - BN / 2, cl - BN / 2);
          uint32_t pk[BN / 4];
#pragma unroll
          for (int e = 0; e < BN / 4; ++e) {
            const float2 x = ffma2(make_float2(sh[2 * e], sh[2 * e + 1]), c2v, nmv);
            const float2 pr = ((kPolyPairs >> e) & 1u) ? exp2_poly2(x)
                                                              : make_float2(ex2_approx(x.x), ex2_approx(x.y));
            if (e & 1) acc1 = fadd2(acc1, pr); else acc0 = fadd2(acc0, pr);
            pk[e] = pack_bf16x2(pr.x, pr.y);
          }
          tmem_st32u(tS + BN / 4, pk);
          tmem_wait_st();
          tc_fence_before();
          if constexpr (PAIR) {
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(C::bar_phi(sb)));
          } else {
            mbar_arrive(bar(C::bar_phi(sb)));
          }
        }
        l = l * alpha + ((acc0.x + acc0.y) + (acc1.x + acc1.y));
        m_use = m_new;
      }
      // Wait for the last P.V.  A parity wait for completion k is only
      // unambiguous once completion k-1 has happened: with two slots the
      // last S_i was issued behind P.V(n-2), with one slot it was not, so
      // there completion n-2 is awaited first.
      bool got_o = ok;
      if (got_o && C::NSLOT == 1 && n_tiles >= 2)
        got_o = mbar_wait(bar(C::bar_pv(0)), (uint32_t)(T + n_tiles - 2) & 1u, wd);
      got_o = got_o && mbar_wait(bar(C::bar_pv(C::NSLOT == 2 ? slot : 0)), (uint32_t)(T + n_tiles - 1) & 1u, wd);
      if (__any_sync(0xffffffffu, !got_o)) {
        ok = false;
      } else {
        tc_fence_after();
        // The sink joins the denominator against a common maximum M, so a
        // large sink logit cannot overflow: O = O_acc 2^(m - M) / l',
        // l' = l 2^(m - M) + 2^(sink - M), LSE = M + log2 l'.
        float m_fin = m_use, inv_l;
        if (MODE != MODE_PLAIN && p.ext.sinks != nullptr) {
          const float s2 = __ldg(p.ext.sinks + h) * 1.4426950408889634f;
          m_fin = fmaxf(m_use, s2);
          const float a = ex2_approx(m_use - m_fin);
          l = l * a + ex2_approx(s2 - m_fin);
          inv_l = a / l;
        } else {
          inv_l = l > 0.f ? 1.f / l : 0.f;
        }
        const bool row_ok = s_row < p.Sq;
        const size_t row_off = (((size_t)x.b * p.Sq + s_row) * p.Hq + h) * (size_t)D;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          float v[32];
          tmem_ld32(tO + 32 * c, v);
          if (row_ok) {
            if (p.out_f32) {
              float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(p.out) + row_off + 32 * c);
#pragma unroll
              for (int q4 = 0; q4 < 8; ++q4)
                dst[q4] = make_float4(v[4 * q4] * inv_l, v[4 * q4 + 1] * inv_l, v[4 * q4 + 2] * inv_l,
                                      v[4 * q4 + 3] * inv_l);
            } else {
              uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(p.out) + row_off + 32 * c);
#pragma unroll
              for (int q8 = 0; q8 < 4; ++q8)
                dst[q8] = make_uint4(pack_bf16x2(v[8 * q8] * inv_l, v[8 * q8 + 1] * inv_l),
                                     pack_bf16x2(v[8 * q8 + 2] * inv_l, v[8 * q8 + 3] * inv_l),
                                     pack_bf16x2(v[8 * q8 + 4] * inv_l, v[8 * q8 + 5] * inv_l),
                                     pack_bf16x2(v[8 * q8 + 6] * inv_l, v[8 * q8 + 7] * inv_l));
            }
          }
        }
        if (row_ok && p.lse != nullptr)
          p.lse[((size_t)x.b * p.Hq + h) * p.Sq + s_row] = l > 0.f ? (m_fin + log2f(l)) * LN2 : -INFINITY;
      }
      // O of this slot may now be overwritten by the next unit's first P.V
      tc_fence_before();
      if constexpr (PAIR) {
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(C::bar_ofree(slot)));
      } else {
        mbar_arrive(bar(C::bar_ofree(slot)));
      }
      T += n_tiles;
    }
    tc_fence_before();
  }

  __syncwarp();
  __syncthreads();
  if (*abort_flag) {
    // Nothing may still write this CTA's shared memory or TMEM when it exits.
    if (warp == C::WARP_PRODUCER && lane == 0) {
      if (q_issued > 0) drain_wait(bar(C::BAR_Q), (uint32_t)(q_issued - 1) & 1u, p.timeout_ns);
    }
    if (MB && warp == C::WARP_PRODUCER && lane == 1 && m_issued > 0) {
      // only the last MSTAGES mask tiles can still be in flight: an earlier
      // one was consumed (after it arrived) before its stage was reloaded
      for (int tg = max(0, m_issued - C::MSTAGES); tg < m_issued; ++tg)
        for (int h = 0; h < 2; ++h)
          drain_wait(bar(C::bar_mfull(tg % C::MSTAGES, h)), (uint32_t)(tg / C::MSTAGES) & 1u, p.timeout_ns);
    }
    if (warp == C::WARP_PRODUCER && lane == 0) {
      for (int n = max(0, issued - C::NBUF); n < issued; ++n)
        drain_wait(bar(C::bar_full(n % C::NBUF)), (uint32_t)(n / C::NBUF) & 1u, p.timeout_ns);
    }
    if (warp == C::WARP_MMA && lane == 0 && (!PAIR || rank == 0)) {
      if constexpr (PAIR) mma_commit_pair(bar(C::BAR_DRAIN));
      else mma_commit(bar(C::BAR_DRAIN));
      drain_wait(bar(C::BAR_DRAIN), 0, p.timeout_ns);
    }
    __syncwarp();
    __syncthreads();
  }
  if constexpr (PAIR) {
    // the leader's MMAs read this CTA's shared memory and write its TMEM:
    // neither CTA frees either before both are done (every wait above is
    // bounded, so both CTAs reach this barrier)
    tc_fence_before();
    cg::this_cluster().sync();
    tc_fence_after();
  }
  if (warp == C::WARP_MMA) {
    tc_fence_after();
    if constexpr (PAIR) tmem_dealloc2(tmem, C::TMEM_COLS);
    else tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

template <int DK, int DV, int MODE>
int launch_t(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tm,
             const PrefillParams& p, cudaStream_t stream) {
  using C = PrefillCfg<DK, DV, MODE == MODE_ALIBI_MASK || MODE == MODE_CAP_MASK>;
  cudaError_t e = cudaFuncSetAttribute(prefill_kernel<DK, DV, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)C::SMEM);
  if (e != cudaSuccess) return (int)e;
  const long long units = (long long)p.n_qt * p.B * p.Hkv * p.units_per_kvh;
  if (units <= 0 || units > 0x7fffffffLL || p.num_ctas <= 0) return (int)cudaErrorInvalidValue;
  const long long grid = units < p.num_ctas ? units : p.num_ctas;  // persistent: one CTA per SM
  prefill_kernel<DK, DV, MODE><<<(unsigned)grid, C::THREADS, C::SMEM, stream>>>(tq, tk, tv, tm, p);
  return (int)cudaGetLastError();
}

// The CTA-pair form: clusters of two CTAs, as many as fit at once (at most
// one per unit); tk64 tiles K in 64-key boxes.
template <int D, int MODE>
int launch_pair_t(const CUtensorMap& tq, const CUtensorMap& tk64, const CUtensorMap& tv, const PrefillParams& p,
                  cudaStream_t stream) {
  using C = PrefillCfg<D, D, false, true>;
  auto kern = prefill_kernel<D, D, MODE, true>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::SMEM);
  if (e != cudaSuccess) return (int)e;
  const long long units = (long long)p.n_qt * p.B * p.Hkv * p.units_per_kvh;
  if (units <= 0 || units > 0x7fffffffLL || p.num_ctas < 2) return (int)cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(C::THREADS);
  cfg.dynamicSmemBytes = C::SMEM;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  long long clusters = p.num_ctas / 2;
  cfg.gridDim = dim3((unsigned)(2 * clusters));
  int fit = 0;
  if (cudaOccupancyMaxActiveClusters(&fit, kern, &cfg) == cudaSuccess && fit > 0 && fit < clusters) clusters = fit;
  (void)cudaGetLastError();   // an occupancy query that failed leaves the grid at one cluster per SM pair
  if (units < clusters) clusters = units;
  cfg.gridDim = dim3((unsigned)(2 * clusters));
  e = cudaLaunchKernelEx(&cfg, kern, tq, tk64, tv, tv, p);
  if (e != cudaSuccess) return (int)e;
  return (int)cudaGetLastError();
}

}  // namespace

int launch_prefill_pair(int D, bool ext, const CUtensorMap& tq, const CUtensorMap& tk64, const CUtensorMap& tv,
                        const PrefillParams& p, cudaStream_t stream) {
  if (D != 256 || p.ext.mask != nullptr || p.g % 2 != 0) return (int)cudaErrorInvalidValue;
  const int mode = !ext ? MODE_PLAIN : p.ext.cap_a > 0.f ? MODE_CAP : p.ext.alibi ? MODE_ALIBI : MODE_MASKS;
  switch (mode) {
    case MODE_PLAIN: return launch_pair_t<256, MODE_PLAIN>(tq, tk64, tv, p, stream);
    case MODE_MASKS: return launch_pair_t<256, MODE_MASKS>(tq, tk64, tv, p, stream);
    case MODE_ALIBI: return launch_pair_t<256, MODE_ALIBI>(tq, tk64, tv, p, stream);
    default: return launch_pair_t<256, MODE_CAP>(tq, tk64, tv, p, stream);
  }
}

size_t prefill_smem_bytes(int D, int Dv) {
  if (D == Dv) {
    switch (D) {
      case 64: return PrefillCfg<64>::SMEM;
      case 128: return PrefillCfg<128>::SMEM;
      case 256: return PrefillCfg<256>::SMEM;
      default: return 0;
    }
  }
  return (D == 192 && Dv == 128) ? PrefillCfg<192, 128>::SMEM : 0;
}

int prefill_slots(int Dv) { return Dv <= 128 ? 2 : 1; }

bool prefill_dims_supported(int D, int Dv) {
  return (D == Dv && (D == 64 || D == 128 || D == 256)) || (D == 192 && Dv == 128);
}

template <int DK, int DV>
int launch_mode(int mode, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tm,
                const PrefillParams& p, cudaStream_t stream) {
  switch (mode) {
    case MODE_PLAIN: return launch_t<DK, DV, MODE_PLAIN>(tq, tk, tv, tm, p, stream);
    case MODE_MASKS: return launch_t<DK, DV, MODE_MASKS>(tq, tk, tv, tm, p, stream);
    case MODE_ALIBI: return launch_t<DK, DV, MODE_ALIBI>(tq, tk, tv, tm, p, stream);
    case MODE_CAP: return launch_t<DK, DV, MODE_CAP>(tq, tk, tv, tm, p, stream);
    case MODE_ALIBI_MASK: return launch_t<DK, DV, MODE_ALIBI_MASK>(tq, tk, tv, tm, p, stream);
    default: return launch_t<DK, DV, MODE_CAP_MASK>(tq, tk, tv, tm, p, stream);
  }
}

int launch_prefill(int D, int Dv, bool ext, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                   const CUtensorMap& tm, const PrefillParams& p, cudaStream_t stream) {
  // the cheapest variant that covers the requested terms
  const int mode = !ext ? MODE_PLAIN
                   : p.ext.cap_a > 0.f ? (p.ext.mask != nullptr ? MODE_CAP_MASK : MODE_CAP)
                   : p.ext.mask != nullptr ? MODE_ALIBI_MASK
                   : p.ext.alibi ? MODE_ALIBI
                   : MODE_MASKS;
  if (D == 192 && Dv == 128) return launch_mode<192, 128>(mode, tq, tk, tv, tm, p, stream);
  if (D != Dv) return (int)cudaErrorInvalidValue;
  switch (D) {
    case 64: return launch_mode<64, 64>(mode, tq, tk, tv, tm, p, stream);
    case 128: return launch_mode<128, 128>(mode, tq, tk, tv, tm, p, stream);
    case 256: return launch_mode<256, 256>(mode, tq, tk, tv, tm, p, stream);
    default: return (int)cudaErrorInvalidValue;
  }
}

}  // namespace gqa
