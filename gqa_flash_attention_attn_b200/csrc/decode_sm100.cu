// Split-KV decode ("flash decoding") for sm_100a, swapped-operand form.
//
// A CTA owns one (split, batch, K/V head).  Its R = g*Sq query rows (all the
// query heads of the group times the Sq draft rows) are the N side of the
// MMAs, so the 128 keys of a tile fill the M = 128 side:
//
//   S^T [128 keys x RP rows]  = K_tile [128 x D] . Q^T        (tcgen05, TMEM)
//   O^T [128 d    x RP rows] += V_tile^T [128 d x 128 keys] . P^T  per 128-d chunk
//
// The softmax warpgroup holds one key per thread (TMEM lane) and reduces each
// row across the 128 keys with warp shuffles plus a cross-warp step in shared
// memory ("Anbeeld/beellama.cpp PR #149", Overview: warp-shuffle reduction,
// fp32 rescale, QB = 8 query rows per block for verify steps).  P is rounded
// to bf16 into a 128-byte-swizzled shared buffer that the next MMA reads.
//
// Every split publishes its normalised partial O and its log-sum-exp, also
// when it has no visible key (lse = -inf, O = 0) ("Anbeeld/beellama.cpp PR
// #149", Overview, ub>64 fix: every block publishes its (max, rowsum)); the
// merge is attn_merge.  Or (cmerge) the splits of one (b, kvh) form a thread-
// block cluster: each CTA leaves its (max, rowsum) and unnormalised O in its
// own shared memory and every CTA merges a slice of the columns from all of
// them over distributed shared memory, writing the final O and LSE, so no
// partial reaches HBM and no second launch runs.
//
// The kernel is HBM-bound, so the pipeline keeps loads flowing while the
// softmax works: S^T and P are double-buffered, the MMA thread computes
// S_{j+1} before it waits for P_j, and the producer streams the ring in the
// same order (K_0, K_1, V_0, K_2, V_1, ...).  Ring slots are 32 KB (128 keys
// x 128 columns, two TMA boxes); two CTAs run per SM.
#include <cooperative_groups.h>

#include "kernels.h"
#include "ptx.cuh"

namespace gqa {
namespace {

namespace cg = cooperative_groups;

constexpr int BN = 128;                        // keys per tile
constexpr uint32_t BOX_BYTES = 128u * 128u;    // 128 rows x 64 bf16
constexpr uint32_t SLOT_BYTES = 2u * BOX_BYTES;
constexpr float LN2 = 0.6931471805599453f;
constexpr int THREADS = 192;                   // warps 0-3 softmax, 4 producer, 5 MMA
constexpr int WARP_PRODUCER = 4;
constexpr int WARP_MMA = 5;
constexpr int MAX_NBUF = 6;
constexpr int MAX_GROUP = 8;                   // consecutive splits per CTA
constexpr int MAX_CLUSTER = 16;                // CTAs of one (b, kvh) merged in a cluster
template <int N>
struct IntC { static constexpr int value = N; };

// One split of a CTA's group: its tiles are first .. first+nt-1 of the CTA's
// tile stream; keys from kbase on a 128-key grid, the split ending at hi.
struct SegInfo {
  int first, nt, kbase, hi;
  int ob, pad0, pad1, pad2;   // ob: the O^T buffer the split accumulates in
};

// Walks a CTA's tile stream in order: the split of tile j in registers,
// reading the shared table only when a split boundary is crossed.
struct SegCursor {
  const SegInfo* tab;
  int n, i, next_first;
  int first, nt, kbase, hi, ob;   // the current split's entry
  __device__ __forceinline__ void load(int k) {
    first = tab[k].first;
    nt = tab[k].nt;
    kbase = tab[k].kbase;
    hi = tab[k].hi;
    ob = tab[k].ob;
    next_first = k + 1 < n ? tab[k + 1].first : 0x7fffffff;
  }
  __device__ __forceinline__ SegCursor(const SegInfo* t, int nseg) : tab(t), n(nseg), i(0) { load(0); }
  // position on tile j (non-decreasing over calls)
  __device__ __forceinline__ void to(int j) {
    while (j >= next_first) load(++i);
  }
  // first key of tile j (its split's tiles reversed under ALiBi)
  __device__ __forceinline__ int key0(int j, bool rev) const {
    const int jj = j - first;
    return kbase + (rev ? nt - 1 - jj : jj) * 128;
  }
};
// A staged mask row: the tile's 128 keys in an 8-key-aligned window of 136
// (17 chunks of 16 bytes), so every cp.async source is 16-byte aligned.
constexpr int MROW_KEYS = 136;
constexpr uint32_t MROW_BYTES = MROW_KEYS * 2u;

struct Layout {
  uint32_t off_q, off_q8, off_p, off_ring, off_red, off_row, off_mask, off_bar, off_misc, off_seg, total;
  // mrows: query rows s whose additive-mask values are staged per tile;
  // fp8: K/V slots of 128 e4m3 columns (16 KB) and Q as two e4m3 planes
  __host__ __device__ Layout(int D, int RP, int nbuf, int mrows, bool fp8) {
    off_q = 0;
    const uint32_t qbytes = (uint32_t)(D / 64) * RP * 128u;
    off_q8 = (off_q + qbytes + 1023u) & ~1023u;
    const uint32_t q8bytes = fp8 ? 2u * (uint32_t)(D / 128) * RP * 128u : 0u;   // hi, lo planes
    off_p = (off_q8 + q8bytes + 1023u) & ~1023u;
    off_ring = (off_p + 2u * 2u * RP * 128u + 1023u) & ~1023u;  // two P buffers
    off_red = off_ring + (uint32_t)nbuf * (fp8 ? BOX_BYTES : SLOT_BYTES);
    off_row = off_red + 2u * 4u * RP * 4u;     // red_max[4][RP], red_sum[4][RP]
    off_mask = off_row + 13u * RP * 4u;        // m, l, alpha, msub, inv, lim, limlo, pos, slope, mask row, thrx, delta
    off_bar = off_mask + (uint32_t)mrows * 2u * MROW_BYTES;  // staged mask [2][mrows][136 keys] bf16
    off_bar = (off_bar + 7u) & ~7u;
    off_misc = off_bar + (uint32_t)(1 + 2 * nbuf + 8) * 8u;
    off_seg = off_misc + 16u;                  // SegInfo[MAX_GROUP]
    total = off_seg + (uint32_t)MAX_GROUP * 32u + 1024u;
  }
};

__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > limit_ns) break;
  }
}

// Reduce 16 per-lane values (one per row) across the 32 lanes of a warp.
// On return, lanes l and l^16 hold the reduction of row (l & 15) in v[0].
// 16 shuffles instead of 16 x 5.
template <bool kMax>
__device__ __forceinline__ float warp_reduce16(float (&v)[16], int lane) {
#pragma unroll
  for (int step = 8; step >= 1; step >>= 1) {
    const bool upper = (lane & step) != 0;
#pragma unroll
    for (int i = 0; i < step; ++i) {
      const float send = upper ? v[i] : v[i + step];
      const float keep = upper ? v[i + step] : v[i];
      const float recv = __shfl_xor_sync(0xffffffffu, send, step);
      v[i] = kMax ? fmaxf(keep, recv) : keep + recv;
    }
  }
  const float other = __shfl_xor_sync(0xffffffffu, v[0], 16);
  return kMax ? fmaxf(v[0], other) : v[0] + other;
}

// Logits in log2 units of this thread's key for the 16 rows 16q..16q+15 with
// the optional terms: softcap or plain scaling, ALiBi slope * (key - pos), and
// the additive mask (staged per tile in shared memory, or read directly).
// Per-row constants come in as 16-byte shared-memory vectors and every term's
// test sits outside the unrolled loops.
__device__ __forceinline__ void ext_rows16(float (&v)[16], const LogitExt& x, float c2, int key, int t, int q,
                                           const float* slope_sm, const int* pos_sm, const uint16_t* mst,
                                           int mask_rows, int q_offset, const uint16_t* const* mrow_sm, int hi) {
  if (x.cap_a > 0.f) {
#pragma unroll
    for (int e = 0; e < 16; ++e) v[e] = x.cap_b * tanh_approx(v[e] * x.cap_a);
  } else {
#pragma unroll
    for (int e = 0; e < 16; ++e) v[e] *= c2;
  }
  if (x.alibi || mask_rows > 0) {
    int ps[16];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int4 w = reinterpret_cast<const int4*>(pos_sm + 16 * q)[i];
      ps[4 * i] = w.x; ps[4 * i + 1] = w.y; ps[4 * i + 2] = w.z; ps[4 * i + 3] = w.w;
    }
    if (x.alibi) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 w = reinterpret_cast<const float4*>(slope_sm + 16 * q)[i];
        v[4 * i] = fmaf(w.x, (float)(key - ps[4 * i]), v[4 * i]);
        v[4 * i + 1] = fmaf(w.y, (float)(key - ps[4 * i + 1]), v[4 * i + 1]);
        v[4 * i + 2] = fmaf(w.z, (float)(key - ps[4 * i + 2]), v[4 * i + 2]);
        v[4 * i + 3] = fmaf(w.w, (float)(key - ps[4 * i + 3]), v[4 * i + 3]);
      }
    }
    if (mask_rows > 0) {
      // mst: this tile's staged mask, already offset to this thread's key
#pragma unroll
      for (int e = 0; e < 16; ++e)
        v[e] = fmaf(__uint_as_float((uint32_t)mst[(ps[e] - q_offset) * MROW_KEYS] << 16), 1.4426950408889634f,
                    v[e]);
    }
  }
  if (x.mask != nullptr && mask_rows == 0) {
    // too many rows to stage: read inside the split only (key < hi <= Skv)
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const uint16_t* mr = mrow_sm[16 * q + e];
      if (mr != nullptr && key < hi)
        v[e] = fmaf(__uint_as_float((uint32_t)__ldg(mr + key) << 16), 1.4426950408889634f, v[e]);
    }
  }
}

// O^T / l of one split from TMEM to the fp32 partial (rows r < R of this
// CTA's group), called once per split: kept out of line so the tile loop
// stays small.  Thread t owns column t of each 128-column chunk (of the one
// 64-column chunk when D = 64: threads 64-127 then hold no column).
template <int D>
__device__ __noinline__ void write_partial_o(uint32_t taddr, int RP, int R, int g, int kvh, int b, int s0, int Sq,
                                             int Hq, void* out, bool out_bf16, const float* inv_sm, int t) {
  constexpr int KC = (D + 127) / 128;
  if (t >= (D < 128 ? D : 128)) return;
  for (int c = 0; c < KC; ++c) {
    for (int q = 0; q < RP / 16; ++q) {
      float v[16];
      tmem_ld16(taddr + (uint32_t)(c * RP + 16 * q), v);
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const int r = 16 * q + e;
        if (r < R) {
          const int s = s0 + r / g, h = kvh * g + (r % g);
          const size_t o = (((size_t)b * Sq + s) * Hq + h) * D + c * 128 + t;
          if (out_bf16)
            reinterpret_cast<__nv_bfloat16*>(out)[o] = __float2bfloat16_rn(v[e] * inv_sm[r]);
          else
            reinterpret_cast<float*>(out)[o] = v[e] * inv_sm[r];
        }
      }
    }
  }
}

// The merge of a cluster's key ranges (cmerge).  CTA rank k holds, for rows
// r < RP, m_k[r] and l_k[r] (log2 units; with fp8 P carries the factor 2^6
// of the tile loop) and X_k[r][d] = v_scale * unnormalised O.  With M =
// max_k m_k (and the sink logit, which joins only M and the denominator),
// w_k = 2^(m_k - M), L = sum_k w_k l_k:  O = sum_k w_k X_k / L and LSE =
// (M + log2 L) ln 2.  Rank c writes columns [c DV/n, (c+1) DV/n) of every
// row, reading them from all n CTAs over distributed shared memory; rank 0
// writes the LSE.  Threads t = 0..127 (named barrier 1).
template <int DV, bool EXT, bool FP8>
__device__ __noinline__ void cluster_merge(const DecodeParams& p, float* m_sm, float* l_sm, float* xbuf, float* wbuf,
                                           int R, int RP, int g, int kvh, int b, int s0, int t) {
  cg::cluster_group cl = cg::this_cluster();
  const int n = (int)cl.num_blocks();
  const int c = (int)cl.block_rank();
  float* inv = wbuf + MAX_CLUSTER * RP;   // 1 / L per row, after the weights W[k][r]
  const float off = FP8 ? 6.f : 0.f;
  for (int r = t; r < RP; r += 128) {
    float sink2 = -INFINITY;
    if (EXT && p.ext.sinks != nullptr && r < R)
      sink2 = __ldg(p.ext.sinks + kvh * g + (r % g)) * 1.4426950408889634f + off;
    float M = sink2;
    for (int k = 0; k < n; ++k) M = fmaxf(M, cl.map_shared_rank(m_sm, k)[r]);
    float L = 0.f;
    for (int k = 0; k < n; ++k) {
      const float mk = cl.map_shared_rank(m_sm, k)[r];
      const float w = (mk == -INFINITY) ? 0.f : ex2_approx(mk - M);
      wbuf[k * RP + r] = w;
      L = fmaf(w, cl.map_shared_rank(l_sm, k)[r], L);
    }
    if (sink2 != -INFINITY) L += ex2_approx(sink2 - M);
    inv[r] = L > 0.f ? 1.f / L : 0.f;
    if (c == 0 && r < R && p.part_lse != nullptr) {
      const int s = s0 + r / g, h = kvh * g + (r % g);
      p.part_lse[((size_t)b * p.Hq + h) * p.Sq + s] = L > 0.f ? (M + log2f(L) - off) * LN2 : -INFINITY;
    }
  }
  named_bar_sync(1, 128);
  const int cols = DV / n;
  const int c0 = c * cols;
  for (int idx = t; idx < R * cols; idx += 128) {
    const int r = idx / cols, d = c0 + (idx - r * cols);
    float acc = 0.f;
    for (int k = 0; k < n; ++k) {
      const float w = wbuf[k * RP + r];
      if (w != 0.f) acc = fmaf(w, cl.map_shared_rank(xbuf, k)[(size_t)r * DV + d], acc);
    }
    const int s = s0 + r / g, h = kvh * g + (r % g);
    const size_t o = (((size_t)b * p.Sq + s) * p.Hq + h) * DV + d;
    if (p.fout_bf16) reinterpret_cast<__nv_bfloat16*>(p.fout)[o] = __float2bfloat16_rn(acc * inv[r]);
    else reinterpret_cast<float*>(p.fout)[o] = acc * inv[r];
  }
}

// CM: the cluster merge (cmerge) variant; the plain kernels carry none of its code.
template <int DK, int DV, bool EXT, bool PAGED, bool FP8, bool CM>
__global__ void __launch_bounds__(THREADS, 2)
    decode_split_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const DecodeParams p) {
  // K tiles are DK columns wide (Q . K over DK), V tiles and O are DV wide;
  // a K tile takes KCK 128-column slots, the last one half filled when DK is
  // an odd multiple of 64 (e.g. 320, 576)
  constexpr int KCK = (DK + 127) / 128;
  constexpr bool KHALF = (DK % 128) != 0;
  // V slots per tile, and O^T chunks of 128 d-rows; DV = 64 fills the first
  // half of one slot (one box), and O^T rows 64-127 of the P.V MMA (which
  // read the slot's unused second box) are never stored
  constexpr int KC = (DV + 127) / 128;
  constexpr bool VHALF = (DV % 128) != 0;
  constexpr int D = DV;          // output width
  static_assert(DK % 64 == 0 && DV % 64 == 0 && (!VHALF || DV == 64) && (!FP8 || (DK == DV && !VHALF)),
                "head sizes");
  const int RP = p.RP, g = p.g, nbuf = p.nbuf;
  const Layout L(DK, RP, nbuf, p.mask_rows, FP8);
  constexpr uint32_t SLOTB = FP8 ? BOX_BYTES : SLOT_BYTES;   // bytes of one 128-column K/V slot

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  float* red_max = reinterpret_cast<float*>(gbase + L.off_red);
  float* red_sum = red_max + 4 * RP;
  float* m_sm = reinterpret_cast<float*>(gbase + L.off_row);
  float* l_sm = m_sm + RP;
  float* alpha_sm = l_sm + RP;
  float* msub_sm = alpha_sm + RP;
  float* inv_sm = msub_sm + RP;
  int* lim_sm = reinterpret_cast<int*>(inv_sm + RP);     // last visible key of row r
  int* limlo_sm = lim_sm + RP;                             // keys <= this are outside the window
  int* pos_sm = limlo_sm + RP;                             // query position of row r
  float* slope_sm = reinterpret_cast<float*>(pos_sm + RP); // ALiBi slope * log2(e) of row r
  const uint16_t** mrow_sm = reinterpret_cast<const uint16_t**>(slope_sm + RP);  // mask row of row r
  // one-pass tile loop: x > thrx_sm[r] moves row r's maximum (-inf while the
  // row has none); delta_sm[r]: the shift of x when it does
  float* thrx_sm = reinterpret_cast<float*>(mrow_sm + RP);
  float* delta_sm = thrx_sm + RP;
  // staged mask: [2 tiles][mask_rows][136 keys] bf16, filled by cp.async one
  // tile ahead by all softmax threads
  const uint32_t mstage_u32 = base + L.off_mask;
  const uint16_t* mstage = reinterpret_cast<const uint16_t*>(gbase + L.off_mask);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + L.off_misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + L.off_misc + 4);
  volatile int* resc_flag = reinterpret_cast<volatile int*>(gbase + L.off_misc + 8);
  auto bar = [&](int i) -> uint32_t { return base + L.off_bar + 8u * (uint32_t)i; };
  const int BAR_Q = 0;
  auto bar_full = [&](int s) { return 1 + s; };
  auto bar_empty = [&](int s) { return 1 + nbuf + s; };
  const int BAR_S0 = 1 + 2 * nbuf;       // s_full[2]
  const int BAR_P0 = BAR_S0 + 2;         // p_full[2]
  const int BAR_PV0 = BAR_S0 + 4;        // pv_done per P buffer [2]
  const int BAR_DRAIN = BAR_S0 + 6;
  const int BAR_Q8 = BAR_S0 + 7;         // fp8: Q planes written

  // a merge launched after this kernel (programmatic dependent launch) may
  // be scheduled as soon as every CTA of this grid has started; it waits for
  // this grid to complete before it reads anything
  griddep_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bkv = blockIdx.y / p.nqc;
  // query chunks in reverse: with a causal mask the last chunks see the most
  // keys, and CTAs launch in grid order, so the longest start first
  const int qc_in = blockIdx.y - bkv * p.nqc;
  const int qc = p.causal ? p.nqc - 1 - qc_in : qc_in;
  const int b = bkv / p.Hkv, kvh = bkv % p.Hkv;
  const int s0 = qc * p.qchunk;               // this CTA's first query row
  const int Sqc = min(p.qchunk, p.Sq - s0);   // and its query rows
  const int Rbox = g * p.qchunk;               // rows the Q box brings (past Sq: zeros)
  const int R = g * Sqc;                       // real rows
  const int mrows = min(p.mask_rows, Sqc);     // staged mask rows
  // this sequence's keys and the position of its first query row
  int Skv = p.Skv, q_offset = p.q_offset;
  long long chunk = p.chunk;
  if (p.seq_lens != nullptr) {
    const int len = __ldg(p.seq_lens + b);
    Skv = min(max(len, 0), p.Skv);
    if (Skv != len && blockIdx.x == 0 && kvh == 0 && threadIdx.x == 0)
      atomicCAS(p.status, kStatusOk, kStatusInvalidArg);
    q_offset = Skv - p.Sq;
    chunk = (Skv + p.num_splits - 1) / p.num_splits;
  }
  if (PAGED) chunk = (chunk + BN - 1) / BN * BN;  // no tile crosses a page
  q_offset += s0;   // this CTA's rows sit at q_offset .. q_offset + Sqc - 1
  // With ALiBi the bias grows toward each query's own position: visiting a
  // split's tiles newest first sets the running maximum on the first tile and
  // spares the O rescales (the tile order does not change the result).
  const bool rev = EXT && p.ext.alibi != 0;
  // This CTA's splits sg0 .. sg0+nseg-1 of (b, kvh) run as one tile stream
  // (same Q, one pipeline); each split's partial is published at its end.
  const int sg0 = blockIdx.x * p.group;
  const int nseg = min(p.group, p.num_splits - sg0);
  SegInfo* seg_sm = reinterpret_cast<SegInfo*>(gbase + L.off_seg);
  int T = 0;  // tiles of the whole stream
  int filled = 0;  // non-empty splits so far: consecutive ones alternate O^T buffers
  for (int i = 0; i < nseg; ++i) {
    const long long lo_ll = (long long)(sg0 + i) * chunk;
    const int lo = (int)min(lo_ll, (long long)Skv);
    const int hi = (int)min(lo_ll + chunk, (long long)Skv);
    const int eff_hi = p.causal ? (int)min((long long)hi, (long long)q_offset + Sqc) : hi;
    // a sliding window hides every key at or before q_offset - window from all rows
    const int eff_lo = (EXT && p.ext.window > 0) ? max(lo, q_offset - p.ext.window + 1) : lo;
    const int kb = lo + ((eff_lo - lo) / BN) * BN;   // first tile, on the split's tile grid
    const int nt = eff_hi > eff_lo ? (eff_hi - kb + BN - 1) / BN : 0;
    if (threadIdx.x == 0) seg_sm[i] = SegInfo{T, nt, kb, hi, p.obuf == 2 ? (filled & 1) : 0, 0, 0, 0};
    filled += nt > 0 ? 1 : 0;
    if (nt == 0 && !CM) {
      // No visible key in this split: publish (-inf, 0) for every row.
      const size_t so = (size_t)(sg0 + i) * p.B * p.Sq * p.Hq * D;
      const size_t sl = (size_t)(sg0 + i) * p.B * p.Hq * p.Sq;
      for (int x = threadIdx.x; x < R * D; x += THREADS) {
        const int r = x / D, d = x - r * D;
        const int s = s0 + r / g, h = kvh * g + (r % g);
        const size_t o = so + (((size_t)b * p.Sq + s) * p.Hq + h) * D + d;
        if (p.fout == nullptr) p.part_out[o] = 0.f;
        else if (p.fout_bf16) reinterpret_cast<__nv_bfloat16*>(p.fout)[o] = __float2bfloat16_rn(0.f);
        else reinterpret_cast<float*>(p.fout)[o] = 0.f;
      }
      for (int r = threadIdx.x; r < R && p.part_lse != nullptr; r += THREADS) {
        const int s = s0 + r / g, h = kvh * g + (r % g);
        p.part_lse[sl + ((size_t)b * p.Hq + h) * p.Sq + s] = -INFINITY;
      }
    }
    T += nt;
  }
  float* xbuf = reinterpret_cast<float*>(gbase + L.off_ring);   // cmerge: X, then the weights
  float* wbuf = xbuf + (size_t)RP * D;
  if (T == 0) {
    if constexpr (CM) {
      // an empty key range still takes part in the cluster's merge, with weight 0
      if (threadIdx.x < RP) {
        m_sm[threadIdx.x] = -INFINITY;
        l_sm[threadIdx.x] = 0.f;
      }
      cg::this_cluster().sync();
      if (threadIdx.x < 128)
        cluster_merge<DV, EXT, FP8>(p, m_sm, l_sm, xbuf, wbuf, R, RP, g, kvh, b, s0, threadIdx.x);
      cg::this_cluster().sync();
    }
    return;
  }
  // split of stream tile j (empty splits share their successor's first tile);
  // for the rare boundary work, the per-tile paths use SegCursor
  auto seg_of = [&](int j) -> int {
    int i = 0;
    while (i + 1 < nseg && j >= seg_sm[i + 1].first) ++i;
    return i;
  };

  // Zero the padding rows of Q (rows Rbox..RP-1 of every 64-column box).
  for (int i = threadIdx.x; i < (DK / 64) * (RP - Rbox) * 32; i += THREADS) {
    const int box = i / ((RP - Rbox) * 32);
    const int w = i - box * (RP - Rbox) * 32;
    reinterpret_cast<uint32_t*>(gbase + L.off_q + (uint32_t)box * RP * 128u + (uint32_t)Rbox * 128u)[w] = 0u;
  }
  if (threadIdx.x < RP) {
    const int r = threadIdx.x;
    m_sm[r] = -INFINITY;
    l_sm[r] = 0.f;
    msub_sm[r] = 0.f;
    thrx_sm[r] = -INFINITY;
    // last visible key of row r (padding rows see none)
    lim_sm[r] = r < R ? (p.causal ? q_offset + r / g : 0x7fffffff) : -1;
    pos_sm[r] = q_offset + (r < R ? r / g : 0);
    limlo_sm[r] = (EXT && p.ext.window > 0) ? pos_sm[r] - p.ext.window : -1;
    slope_sm[r] = (EXT && p.ext.alibi && r < R)
                      ? alibi_slope_log2e(kvh * g + (r - (r / g) * g), p.ext.l2m0, p.ext.l2m1, p.ext.n2)
                      : 0.f;
    mrow_sm[r] = (EXT && p.ext.mask != nullptr && r < R)
                     ? p.ext.mask + (size_t)b * p.ext.mask_sb + (size_t)(s0 + r / g) * p.ext.mask_sr
                     : nullptr;
  }
  if (threadIdx.x == 0) {
    mbar_init(bar(BAR_Q), 1);
    for (int s = 0; s < nbuf; ++s) {
      mbar_init(bar(bar_full(s)), 1);
      mbar_init(bar(bar_empty(s)), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(BAR_S0 + i), 1);
      mbar_init(bar(BAR_P0 + i), 128);
      mbar_init(bar(BAR_PV0 + i), 1);
    }
    mbar_init(bar(BAR_DRAIN), 1);
    mbar_init(bar(BAR_Q8), 1);
    *abort_flag = 0;
    *resc_flag = 0;
    fence_mbar_init();
  }
  uint32_t tmem_cols = 32;
  while (tmem_cols < (uint32_t)(RP * (2 + p.obuf * KC))) tmem_cols <<= 1;
  if (warp == WARP_MMA) {
    tmem_alloc(smem_u32(tmem_slot), tmem_cols);
    tmem_relinquish();
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  auto TS = [&](int buf) { return (uint32_t)(RP * buf); };            // S^T buffers
  auto TO = [&](int c, int ob) { return (uint32_t)(RP * (2 + ob * KC + c)); };  // O^T chunk c, buffer ob
  auto PB = [&](int buf) { return L.off_p + (uint32_t)buf * 2u * RP * 128u; };  // P buffers
  const Watchdog wd{abort_flag, p.status, p.timeout_ns};
  int issued = 0;

  if (warp == WARP_PRODUCER) {
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      mbar_arrive_expect_tx(bar(BAR_Q), (uint32_t)(DK / 64) * Rbox * 128u);
      for (int kb = 0; kb < DK / 64; ++kb)
        tma_load_4d(base + L.off_q + (uint32_t)kb * RP * 128u, &tm_q, bar(BAR_Q), kb * 64, kvh * g, s0, b);
      // ring order: K_0, then (K_{j+1}, V_j) for j = 0..n-1; KC slots each
      bool ok = true;
      const uint64_t pol_k = p.kv_shared ? l2_policy_evict_last() : l2_policy_evict_normal();
      const uint64_t pol_v = p.kv_shared ? l2_policy_evict_first() : l2_policy_evict_normal();
      int n = 0;
      SegCursor ck(seg_sm, nseg), cv(seg_sm, nseg);   // the K and the V stream
      auto issue = [&](const CUtensorMap* tm, int j, SegCursor& cu) {
        cu.to(j);
        const int key0 = cu.key0(j, rev);
        const bool is_k = tm == &tm_k;
        const int nslot = is_k ? KCK : KC;
        for (int c = 0; c < nslot; ++c, ++n) {
          // K columns at or past DV are never read again as V
          const uint64_t pol = (is_k && c * 128 < DV) ? pol_k : pol_v;
          const int slot = n % nbuf, use = n / nbuf;
          if (use > 0 && !mbar_wait(bar(bar_empty(slot)), (uint32_t)(use - 1) & 1u, wd)) {
            ok = false;
            return;
          }
          // a half-filled last K slot (DK an odd multiple of 64) takes one
          // box, and so does the V slot when DV = 64
          const bool half = (KHALF && is_k && c == KCK - 1) || (VHALF && !is_k);
          mbar_arrive_expect_tx(bar(bar_full(slot)), half ? BOX_BYTES : SLOTB);
          const uint32_t dst = base + L.off_ring + (uint32_t)slot * SLOTB;
          if constexpr (!PAGED) {
            if (FP8) {
              tma_load_4d_hint(dst, tm, bar(bar_full(slot)), c * 128, kvh, key0, b, pol);   // 128 e4m3 columns
            } else {
              tma_load_4d_hint(dst, tm, bar(bar_full(slot)), (2 * c) * 64, kvh, key0, b, pol);
              if (!half) tma_load_4d_hint(dst + BOX_BYTES, tm, bar(bar_full(slot)), (2 * c + 1) * 64, kvh, key0, b, pol);
            }
          } else {
            // paged: each page-sized run of keys from its physical page (the
            // tensor map's outer dimensions are row-in-page and page); a
            // logical page past the table reads as zeros (page -1)
            const int* bt = p.block_table + (size_t)b * p.max_pages;
            const int ps = p.page_size, rows = ps < BN ? ps : BN;
            for (int sub = 0; sub < BN / rows; ++sub) {
              const int key = key0 + sub * rows;
              const int lp = key / ps;
              const int page = lp < p.max_pages ? __ldg(bt + lp) : -1;
              const uint32_t off = (uint32_t)(sub * rows) * 128u;
              if (FP8) {
                tma_load_4d_hint(dst + off, tm, bar(bar_full(slot)), c * 128, kvh, key - lp * ps, page, pol);
              } else {
                tma_load_4d_hint(dst + off, tm, bar(bar_full(slot)), (2 * c) * 64, kvh, key - lp * ps, page, pol);
                if (!half)
                  tma_load_4d_hint(dst + BOX_BYTES + off, tm, bar(bar_full(slot)), (2 * c + 1) * 64, kvh, key - lp * ps,
                              page, pol);
              }
            }
          }
          issued = n + 1;
        }
      };
      issue(&tm_k, 0, ck);
      for (int j = 0; ok && j < T; ++j) {
        if (j + 1 < T) issue(&tm_k, j + 1, ck);
        if (ok) issue(&tm_v, j, cv);
      }
    }
  } else if (warp == WARP_MMA) {
    if (lane == 0) {
      const uint32_t idesc_s = FP8 ? idesc_e4m3_f32(128, RP, false, false) : idesc_bf16_f32(128, RP, false, false);
      const uint32_t idesc_o = FP8 ? idesc_e4m3_f32(128, RP, true, false) : idesc_bf16_f32(128, RP, true, false);
      // fp8: the softmax warps turn Q into two e4m3 planes first
      bool ok = mbar_wait(bar(FP8 ? BAR_Q8 : BAR_Q), 0, wd);
      tc_fence_after();
      int n = 0;
      // S^T_j = K_j Q^T into S buffer j%2, one 128-column slot at a time
      auto mma_s = [&](int j) {
        for (int c = 0; c < KCK; ++c, ++n) {
          const int slot = n % nbuf;
          if (!mbar_wait(bar(bar_full(slot)), (uint32_t)(n / nbuf) & 1u, wd)) { ok = false; return; }
          tc_fence_after();
          const uint32_t kb = base + L.off_ring + (uint32_t)slot * SLOTB;
          if constexpr (FP8) {
            // K rows of 128 e4m3 (one 128-byte swizzled row); Q as hi + lo
            // planes: S^T = K Q_hi^T + K Q_lo^T, 32 columns per MMA
#pragma unroll
            for (int pl = 0; pl < 2; ++pl) {
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const uint32_t a = kb + (uint32_t)kk * 32u;
                const uint32_t qb = base + L.off_q8 + (uint32_t)(pl * KC + c) * RP * 128u + (uint32_t)kk * 32u;
                mma_ss_f8(tmem + TS(j & 1), sdesc_sw128(a, 16, 1024), sdesc_sw128(qb, 16, 1024), idesc_s,
                          (c > 0 || pl > 0 || kk > 0) ? 1u : 0u);
              }
            }
          } else {
            // 16 columns per MMA: 8 per full slot, 4 for a half-filled last K slot
            const int nkk = (KHALF && c == KCK - 1) ? 4 : 8;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              if (kk >= nkk) break;
              const uint32_t in_box = (uint32_t)(kk & 3) * 32u;
              const uint32_t a = kb + (uint32_t)(kk >> 2) * BOX_BYTES + in_box;
              const uint32_t qb = base + L.off_q + (uint32_t)(2 * c + (kk >> 2)) * RP * 128u + in_box;
              mma_ss(tmem + TS(j & 1), sdesc_sw128(a, 16, 1024), sdesc_sw128(qb, 16, 1024), idesc_s,
                     (c > 0 || kk > 0) ? 1u : 0u);
            }
          }
          mma_commit(bar(bar_empty(slot)));
        }
        mma_commit(bar(BAR_S0 + (j & 1)));
      };
      if (ok) mma_s(0);
      SegCursor cpv(seg_sm, nseg);
      for (int j = 0; ok && j < T; ++j) {
        // S buffer (j+1)%2 was last read by softmax j-1, whose P the PV of
        // tile j-1 (issued before this point) already waited for.
        if (j + 1 < T) {
          mma_s(j + 1);
          if (!ok) break;
        }
        if (!mbar_wait(bar(BAR_P0 + (j & 1)), (uint32_t)(j >> 1) & 1u, wd)) { ok = false; break; }
        tc_fence_after();
        // O^T(c) += V_j^T(c) P_j^T; a split's first tile starts O afresh (the
        // softmax read the previous split's O before it handed over P_j)
        cpv.to(j);
        const uint32_t acc0 = (j == cpv.first) ? 0u : 1u;
        for (int c = 0; ok && c < KC; ++c, ++n) {
          const int slot = n % nbuf;
          if (!mbar_wait(bar(bar_full(slot)), (uint32_t)(n / nbuf) & 1u, wd)) { ok = false; break; }
          tc_fence_after();
          const uint32_t vb = base + L.off_ring + (uint32_t)slot * SLOTB;
          if constexpr (FP8) {
            // V^T (MN-major: a 128-byte row holds 128 d-columns of one key),
            // 32 keys per MMA; P^T as hi + lo planes of 128 keys per row
#pragma unroll
            for (int pl = 0; pl < 2; ++pl) {
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const uint32_t a = vb + (uint32_t)kk * 4096u;
                const uint32_t pb = base + PB(j & 1) + (uint32_t)pl * RP * 128u + (uint32_t)kk * 32u;
                mma_ss_f8(tmem + TO(c, cpv.ob), sdesc_sw128(a, BOX_BYTES, 1024), sdesc_sw128(pb, 16, 1024), idesc_o,
                          (acc0 || pl > 0 || kk > 0) ? 1u : 0u);
              }
            }
          } else {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint32_t a = vb + (uint32_t)kk * 2048u;
              const uint32_t pb = base + PB(j & 1) + (uint32_t)(kk >> 2) * RP * 128u + (uint32_t)(kk & 3) * 32u;
              mma_ss(tmem + TO(c, cpv.ob), sdesc_sw128(a, BOX_BYTES, 1024), sdesc_sw128(pb, 16, 1024), idesc_o,
                     (acc0 || kk > 0) ? 1u : 0u);
            }
          }
          mma_commit(bar(bar_empty(slot)));
        }
        if (!ok) break;
        mma_commit(bar(BAR_PV0 + (j & 1)));
      }
    }
  } else {
    // ---- softmax: thread t <-> key t of the tile (TMEM lane t) ----
    const int t = threadIdx.x;          // 0..127
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    float c2 = p.c2;          // logit scale * log2(e) (times the K scale with fp8 K/V)
    LogitExt xe = p.ext;      // the optional terms (softcap rescaled with fp8 K/V)
    float vs = 1.f;           // V scale applied in the epilogue
    bool ok = true;
    if constexpr (FP8) {
      // Q -> two e4m3 planes, hi and lo, of q * qs with qs a power of two that
      // puts max |q| in [128, 256): hi + lo holds every bf16 value exactly
      // (4 + 4 significant bits) unless it underflows below 2^-17 of max |q|.
      // The MMAs then give K_code . (q * qs); the logit scale takes
      // k_scale / qs.
      const bool got_q = mbar_wait(bar(BAR_Q), 0, wd);
      if (named_bar_or(1, 128, !got_q)) {
        ok = false;
      } else {
        tc_fence_after();
        const int cpr = DK / 8;   // 16-byte chunks of 8 bf16 per row
        auto qoff = [&](int r, int col) -> uint32_t {
          return (uint32_t)(col >> 6) * RP * 128u + (uint32_t)r * 128u + ((uint32_t)(((col & 63) >> 3) ^ (r & 7)) << 4);
        };
        float amax = 0.f;
        for (int i = t; i < RP * cpr; i += 128) {
          const int r = i / cpr, col = (i - r * cpr) * 8;
          const uint4 w = *reinterpret_cast<const uint4*>(gbase + L.off_q + qoff(r, col));
          const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int k = 0; k < 4; ++k)
            amax = fmax3(amax, fabsf(__uint_as_float(ww[k] << 16)), fabsf(__uint_as_float(ww[k] & 0xffff0000u)));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        if (lane == 0) red_sum[warp] = amax;
        named_bar_sync(1, 128);
        const float qmax = fmaxf(fmaxf(red_sum[0], red_sum[1]), fmaxf(red_sum[2], red_sum[3]));
        const int ex = max((__float_as_int(qmax) >> 23) - 127, -120);
        const float qs = qmax > 0.f ? __int_as_float((127 + 7 - ex) << 23) : 1.f;
        for (int i = t; i < RP * cpr; i += 128) {
          const int r = i / cpr, col = (i - r * cpr) * 8;
          const uint4 w = *reinterpret_cast<const uint4*>(gbase + L.off_q + qoff(r, col));
          const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
          uint32_t hi[2], lo[2];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float x0 = __uint_as_float(ww[k] << 16) * qs, x1 = __uint_as_float(ww[k] & 0xffff0000u) * qs;
            const uint32_t h = e4m3x2_from(x0, x1);
            const float2 bk = e4m3x2_value(h);
            const uint32_t l = e4m3x2_from(x0 - bk.x, x1 - bk.y);
            hi[k >> 1] = (k & 1) ? (hi[k >> 1] | (h << 16)) : h;
            lo[k >> 1] = (k & 1) ? (lo[k >> 1] | (l << 16)) : l;
          }
          const int c8 = col & 127;
          const uint32_t o8 = (uint32_t)(col >> 7) * RP * 128u + (uint32_t)r * 128u +
                              ((uint32_t)((c8 >> 4) ^ (r & 7)) << 4) + (uint32_t)(c8 & 15);
          *reinterpret_cast<uint2*>(gbase + L.off_q8 + o8) = make_uint2(hi[0], hi[1]);
          *reinterpret_cast<uint2*>(gbase + L.off_q8 + (uint32_t)KC * RP * 128u + o8) = make_uint2(lo[0], lo[1]);
        }
        fence_proxy_async_smem();
        named_bar_sync(1, 128);
        if (t == 0) mbar_arrive(bar(BAR_Q8));
        const float kq = __ldg(p.k_scale + kvh) / qs;
        c2 *= kq;
        if (xe.cap_a > 0.f) xe.cap_a *= kq;
        vs = __ldg(p.v_scale + kvh);
      }
    }
    // Publishing split si of the group: stats() turns its (max, sum) into the
    // LSE and 1/l (rows t < RP, from shared memory: needs no wait), write_o()
    // stores O^T / l from its TMEM buffer (after its last P.V completed).
    auto stats = [&](int si) {
      if (t < RP) {
        float l = l_sm[t];
        float m = m_sm[t];
        if (EXT && p.fout != nullptr && p.ext.sinks != nullptr && t < R) {
          // final output (one split, no merge): fold the sink in against a
          // common maximum, as the merge would
          const float s2 = __ldg(p.ext.sinks + kvh * g + (t % g)) * 1.4426950408889634f + (FP8 ? 6.f : 0.f);
          const float mf = fmaxf(m, s2);
          const float a = ex2_approx(m - mf);
          l = l * a + ex2_approx(s2 - mf);
          inv_sm[t] = vs * a / l;
          m = mf;
        } else {
          inv_sm[t] = l > 0.f ? vs / l : 0.f;
        }
        if (t < R && p.part_lse != nullptr) {
          const int s = s0 + t / g, h = kvh * g + (t % g);
          const size_t sl = (size_t)(sg0 + si) * p.B * p.Hq * p.Sq;
          p.part_lse[sl + ((size_t)b * p.Hq + h) * p.Sq + s] =
              l > 0.f ? (m + log2f(l) - (FP8 ? 6.f : 0.f)) * LN2 : -INFINITY;
        }
      }
    };
    auto write_o = [&](int si) {
      named_bar_sync(1, 128);   // inv_sm of every row
      const size_t so = (size_t)(sg0 + si) * p.B * p.Sq * p.Hq * D;
      // partials (fp32), or with one split the final output itself
      void* dst = p.fout != nullptr ? p.fout : static_cast<void*>(p.part_out + so);
      write_partial_o<D>(tmem + lane_off + TO(0, seg_sm[si].ob), RP, R, g, kvh, b, s0, p.Sq, p.Hq, dst,
                          p.fout != nullptr && p.fout_bf16, inv_sm, t);
      named_bar_sync(1, 128);   // every row's inv_sm read before stats() rewrites it
    };
    // wait (jointly) for the P.V of stream tile j
    auto pv_done = [&](int j) -> bool {
      const bool got = mbar_wait(bar(BAR_PV0 + (j & 1)), (uint32_t)(j >> 1) & 1u, wd);
      if (named_bar_or(1, 128, !got)) return false;
      tc_fence_after();
      return true;
    };
    // With two O^T buffers a finished split's O is written out one tile
    // later (after the next hand-off of P, off the critical path), when the
    // P-buffer wait has shown its last P.V complete: pend / pend_last.
    int pend = -1, pend_last = -1;
    SegCursor cs(seg_sm, nseg), cm(seg_sm, nseg);   // this tile; the mask stage's tile
    // stage tile j+1's mask rows (and tile 0's first) with cp.async; the
    // copies stay in flight across tile j's barriers, and tile j's are
    // complete (and, after the next CTA barrier, visible) before use
    // P of rows 16q..16q+15 at this thread's key (p values in v) into P
    // buffer sb: bf16, or e4m3 hi + lo planes
    auto store_p16 = [&](int sb, int q, float (&v)[16]) {
      const int half = t >> 6, tt = t & 63;
      uint8_t* pcol = gbase + PB(sb) + (size_t)half * RP * 128 + (size_t)(tt & 7) * 2;
      const int chunk16 = tt >> 3;
      if constexpr (!FP8) {
        // bf16 P, one 32-bit word (keys t & ~1, t | 1) per store: for
        // each pair of rows the even lane writes the even row and the odd
        // lane the odd row, each taking its neighbour's value by shuffle
        const bool odd = (t & 1) != 0;
        uint8_t* pword = pcol - (size_t)(tt & 1) * 2;
#pragma unroll
        for (int e = 0; e < 16; e += 2) {
          const float other = __shfl_xor_sync(0xffffffffu, odd ? v[e] : v[e + 1], 1);
          const int r = 16 * q + e + (odd ? 1 : 0);
          const uint32_t w = odd ? pack_bf16x2(other, v[e + 1]) : pack_bf16x2(v[e], other);
          *reinterpret_cast<uint32_t*>(pword + (size_t)r * 128 + ((chunk16 ^ (r & 7)) << 4)) = w;
        }
      }
      if constexpr (FP8) {
        // P as hi + lo e4m3 planes (row r: 128 keys, one 128-byte
        // swizzled row per plane).  A lane holds one key of 4 rows; a
        // 4 x 4 byte transpose in each quad of lanes (two shuffle stages,
        // both planes in one word) gives lane j the 4 keys of row e + j,
        // so every store is a 32-bit word.
        const int j4 = t & 3;
        uint8_t* p8 = gbase + PB(sb) + ((t & 15) & ~3);
        const int ck = t >> 4;
#pragma unroll
        for (int e = 0; e < 16; e += 4) {
          const uint32_t h01 = e4m3x2_from(v[e], v[e + 1]);
          const uint32_t h23 = e4m3x2_from(v[e + 2], v[e + 3]);
          const float2 b01 = e4m3x2_value(h01);
          const float2 b23 = e4m3x2_value(h23);
          const uint32_t l01 = e4m3x2_from(v[e] - b01.x, v[e + 1] - b01.y);
          const uint32_t l23 = e4m3x2_from(v[e + 2] - b23.x, v[e + 3] - b23.y);
          uint32_t H = h01 | (h23 << 16), Lw = l01 | (l23 << 16);   // byte i: row e + i
          // stage 1 (lanes j, j ^ 1): even lanes end with rows e, e+2 and
          // odd lanes with rows e+1, e+3, each for keys (j & ~1, j | 1)
          {
            const uint32_t snd = (j4 & 1) ? __byte_perm(H, Lw, 0x6420) : __byte_perm(H, Lw, 0x7531);
            const uint32_t rcv = __shfl_xor_sync(0xffffffffu, snd, 1);
            if (j4 & 1) {
              H = __byte_perm(H, rcv, 0x3514);
              Lw = __byte_perm(Lw, rcv, 0x3716);
            } else {
              H = __byte_perm(H, rcv, 0x5240);
              Lw = __byte_perm(Lw, rcv, 0x7260);
            }
          }
          // stage 2 (lanes j, j ^ 2): lane j ends with row e + j, keys 0-3
          {
            const uint32_t snd = (j4 & 2) ? __byte_perm(H, Lw, 0x5410) : __byte_perm(H, Lw, 0x7632);
            const uint32_t rcv = __shfl_xor_sync(0xffffffffu, snd, 2);
            if (j4 & 2) {
              H = __byte_perm(H, rcv, 0x3254);
              Lw = __byte_perm(Lw, rcv, 0x3276);
            } else {
              H = __byte_perm(H, rcv, 0x5410);
              Lw = __byte_perm(Lw, rcv, 0x7610);
            }
          }
          const int r = 16 * q + e + j4;
          const uint32_t o = (uint32_t)r * 128u + ((uint32_t)(ck ^ (r & 7)) << 4);
          *reinterpret_cast<uint32_t*>(p8 + o) = H;
          *reinterpret_cast<uint32_t*>(p8 + (uint32_t)RP * 128u + o) = Lw;
        }
      }
    };
    auto stage_masks = [&](int j) {
      if (!(EXT && p.mask_rows > 0)) return;
      auto stage = [&](int jj) {
        cm.to(jj);
        const int tile_al = cm.key0(jj, rev) & ~7;
        const int shi = cm.hi;
        const uint32_t dst0 = mstage_u32 + (uint32_t)(jj & 1) * p.mask_rows * MROW_BYTES;
        for (int c = t; c < mrows * 17; c += 128) {
          const int row = c / 17, k8 = (c - row * 17) * 8;
          const int key8 = tile_al + k8;
          const int n = min(max(shi - key8, 0), 8);   // keys inside the split (end <= Skv)
          const uint16_t* src = n > 0 ? p.ext.mask + (size_t)b * p.ext.mask_sb + (size_t)(s0 + row) * p.ext.mask_sr + key8
                                      : p.ext.mask;
          cp_async16(dst0 + (uint32_t)row * MROW_BYTES + (uint32_t)k8 * 2u, src, (uint32_t)n * 2u);
        }
        cp_async_commit();
      };
      if (j == 0) stage(0);
      if (j + 1 < T) {
        stage(j + 1);
        cp_async_wait<1>();
      } else {
        cp_async_wait<0>();
      }
    };
    bool one_pass_done = false;
    if constexpr (FP8 || EXT) {
      if (RP <= 32) {
      // One pass per tile for up to 32 rows (one or two groups of 16 held in
      // registers), for the variants whose softmax outweighs a tile's load:
      // fp8 K/V (half the bytes per tile) and the optional logit terms.  (The
      // plain bf16 kernels keep the two-pass loop below: there the tile
      // stream is paced by the K/V ring, and an earlier hand-off of P only
      // moved the MMA thread's waits, measured 5 % slower on the 8-row verify
      // decode.)  Each logit is taken relative to its row's subtrahend
      // msub (x = logit - msub, log2 units; p = 2^x) and checked against the
      // stale-maximum threshold on the spot: x > 8 is a logit more than 8
      // (bf16 P) or 2 (fp8 P, stored as 64 p: msub = m - 6) above the row's
      // running maximum m.  Only a tile where that happens runs the
      // row-maximum reduction; the rule is the one of the two-pass loop
      // below, so P is the same.  Row sums stay per thread (key) until the
      // split ends, where one reduction gives l.
      auto one_pass = [&](auto nq_tag) {
        constexpr int NQ = decltype(nq_tag)::value;
        constexpr float OFF = FP8 ? 6.f : 0.f;
        float lacc[NQ][16];
#pragma unroll
        for (int q = 0; q < NQ; ++q)
#pragma unroll
          for (int e = 0; e < 16; ++e) lacc[q][e] = 0.f;
        // the split's row sums into l_sm (rows t < RP); partial sums restart
        auto reduce_l = [&]() {
#pragma unroll
          for (int q = 0; q < NQ; ++q) {
            float v[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              v[e] = lacc[q][e];
              lacc[q][e] = 0.f;
            }
            const float x = warp_reduce16<false>(v, lane);
            if (lane < 16) red_sum[warp * RP + 16 * q + lane] = x;
          }
          named_bar_sync(1, 128);
          if (t < RP) l_sm[t] = (red_sum[t] + red_sum[RP + t]) + (red_sum[2 * RP + t] + red_sum[3 * RP + t]);
        };
        for (int j = 0; ok && j < T; ++j) {
          const int sb = j & 1;
          cs.to(j);
          const int jl = j - cs.first;   // tile within its split
          const int hi = cs.hi;           // the split's end key
          if (jl == 0 && j > 0) {
            // a new split: publish the previous one (as in the loop below),
            // then restart its rows
            if (pend >= 0) {
              if (!pv_done(pend_last)) { ok = false; break; }
              write_o(pend);
              pend = -1;
            }
            const int prev = seg_of(j - 1);
            reduce_l();
            stats(prev);
            if (t < RP) {
              m_sm[t] = -INFINITY;
              msub_sm[t] = 0.f;
              thrx_sm[t] = -INFINITY;
            }
            named_bar_sync(1, 128);   // the restarted rows, before any thread reads them
            if (p.obuf == 2) {
              pend = prev;
              pend_last = j - 1;
            } else {
              if (!pv_done(j - 1)) { ok = false; break; }
              write_o(prev);
            }
          }
          stage_masks(j);
          const bool got_s = mbar_wait(bar(BAR_S0 + sb), (uint32_t)(j >> 1) & 1u, wd);
          // A staged mask needs a CTA barrier to be visible; otherwise a give-up
          // here only has to be warp-uniform (TMEM loads are warp-collective),
          // and the joint vote below takes it.
          const bool fail_s =
              (EXT && p.mask_rows > 0) ? named_bar_or(1, 128, !got_s) : __any_sync(0xffffffffu, !got_s);
          const int tile0 = cs.key0(j, rev);
          const int key = tile0 + t;
          const uint16_t* mtile = mstage + (size_t)(j & 1) * p.mask_rows * MROW_KEYS + (tile0 & 7) + t;
          const bool full = (tile0 + BN - 1 < hi) && (!p.causal || tile0 + BN - 1 <= q_offset) &&
                            (!EXT || p.ext.window == 0 || tile0 >= q_offset + Sqc - p.ext.window);
          auto visible = [&](int r) -> bool {
            return key < hi && key <= lim_sm[r] && (!EXT || key > limlo_sm[r]);
          };
          float x[NQ][16];
          bool exceed = false;
          if (!fail_s) {
            tc_fence_after();
#pragma unroll
            for (int q = 0; q < NQ; ++q) {
              tmem_ld16(tmem + lane_off + TS(sb) + 16 * q, x[q]);
              if (EXT) ext_rows16(x[q], xe, c2, key, t, q, slope_sm, pos_sm, mtile, mrows, q_offset, mrow_sm, hi);
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const float4 ms = reinterpret_cast<const float4*>(msub_sm + 16 * q)[i];
                const float4 th = reinterpret_cast<const float4*>(thrx_sm + 16 * q)[i];
                const float msv[4] = {ms.x, ms.y, ms.z, ms.w};
                const float thv[4] = {th.x, th.y, th.z, th.w};
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                  const int e = 4 * i + k;
                  float xv = EXT ? x[q][e] - msv[k] : fmaf(x[q][e], c2, -msv[k]);
                  if (!full && !visible(16 * q + e)) xv = -INFINITY;
                  exceed = exceed || xv > thv[k];
                  x[q][e] = xv;
                }
              }
            }
          }
          // P buffer sb was read by the P.V of tile j-2: wait for it before rewriting
          const bool got_pb = (j < 2) || mbar_wait(bar(BAR_PV0 + sb), (uint32_t)((j - 2) >> 1) & 1u, wd);
          const bool fail = fail_s || !got_pb;
          if (named_bar_or(1, 128, fail || exceed)) {
            if (named_bar_or(1, 128, fail)) { ok = false; break; }
            // some row's maximum moves: the tile's row maxima of x
#pragma unroll
            for (int q = 0; q < NQ; ++q) {
              float v[16];
#pragma unroll
              for (int e = 0; e < 16; ++e) v[e] = x[q][e];
              const float mx = warp_reduce16<true>(v, lane);
              if (lane < 16) red_max[warp * RP + 16 * q + lane] = mx;
            }
            named_bar_sync(1, 128);
            if (t < RP) {
              const float mx =
                  fmaxf(fmaxf(red_max[t], red_max[RP + t]), fmaxf(red_max[2 * RP + t], red_max[3 * RP + t]));
              float delta = 0.f, alpha = 1.f;
              if (mx > thrx_sm[t]) {
                // the row's new maximum m' = msub + mx: msub' = m' - OFF and
                // x' = x + delta with delta = OFF - mx; O and l scale by
                // 2^(m - m') = 2^delta (0 while m was -inf)
                delta = OFF - mx;
                alpha = (m_sm[t] == -INFINITY) ? 0.f : ex2_approx(delta);
                const float ms = msub_sm[t] - delta;
                msub_sm[t] = ms;
                m_sm[t] = ms + OFF;
                thrx_sm[t] = 8.f;
              }
              delta_sm[t] = delta;
              alpha_sm[t] = alpha;
            }
            named_bar_sync(1, 128);
#pragma unroll
            for (int q = 0; q < NQ; ++q)
#pragma unroll
              for (int e = 0; e < 16; ++e) {
                x[q][e] += delta_sm[16 * q + e];
                lacc[q][e] *= alpha_sm[16 * q + e];
              }
            if (jl > 0) {
              // O^T is accumulated by the P.V of tile j-1: it must have completed
              const bool got_o = mbar_wait(bar(BAR_PV0 + (sb ^ 1)), (uint32_t)((j - 1) >> 1) & 1u, wd);
              if (named_bar_or(1, 128, !got_o)) { ok = false; break; }
              tc_fence_after();
              for (int c = 0; c < KC; ++c) {
#pragma unroll
                for (int q = 0; q < NQ; ++q) {
                  float v[16];
                  const uint32_t addr = tmem + lane_off + TO(c, cs.ob) + 16 * q;
                  tmem_ld16(addr, v);
                  uint32_t u[16];
#pragma unroll
                  for (int e = 0; e < 16; ++e) u[e] = __float_as_uint(v[e] * alpha_sm[16 * q + e]);
                  tmem_st16(addr, u);
                }
              }
            }
          }
          // exponentials, per-thread row sums, P into the B-operand buffer
#pragma unroll
          for (int q = 0; q < NQ; ++q) {
            float v[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              v[e] = ex2_approx(x[q][e]);
              lacc[q][e] += v[e];
            }
            store_p16(sb, q, v);
          }
          fence_proxy_async_smem();
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(bar(BAR_P0 + sb));
          if (pend >= 0 && j >= 2 && pend_last <= j - 2) {
            write_o(pend);
            pend = -1;
          }
        }
        if (ok) reduce_l();
      };
      if (RP <= 16) one_pass(IntC<1>{});
      else one_pass(IntC<2>{});
      one_pass_done = true;
      }
    }
    if (!one_pass_done)
    for (int j = 0; ok && j < T; ++j) {
      const int sb = j & 1;
      cs.to(j);
      const int jl = j - cs.first;   // tile within its split
      const int hi = cs.hi;           // the split's end key
      if (jl == 0 && j > 0) {
        // a new split: publish the previous one, then restart the running
        // (max, sum).  With one O^T buffer its O is read now, before this
        // split's first P.V (which waits for P_j) overwrites it.
        if (pend >= 0) {   // the split before had a single tile: flush it first
          if (!pv_done(pend_last)) { ok = false; break; }
          write_o(pend);
          pend = -1;
        }
        const int prev = seg_of(j - 1);
        stats(prev);
        if (p.obuf == 2) {
          pend = prev;
          pend_last = j - 1;
        } else {
          if (!pv_done(j - 1)) { ok = false; break; }
          write_o(prev);
        }
        if (t < RP) {
          m_sm[t] = -INFINITY;
          l_sm[t] = 0.f;
        }
      }
      // every give-up is decided jointly (barrier + OR) so no thread is left
      // waiting at a named barrier or inside a warp-collective TMEM access
      stage_masks(j);
      const bool got_s = mbar_wait(bar(BAR_S0 + sb), (uint32_t)(j >> 1) & 1u, wd);
      if (named_bar_or(1, 128, !got_s)) { ok = false; break; }
      tc_fence_after();
      const int tile0 = cs.key0(j, rev);
      const int key = tile0 + t;
      // this tile's staged mask at this thread's key
      const uint16_t* mtile = mstage + (size_t)(j & 1) * p.mask_rows * MROW_KEYS + (tile0 & 7) + t;
      // whole tile visible to every real row: no per-element mask
      const bool full = (tile0 + BN - 1 < hi) && (!p.causal || tile0 + BN - 1 <= q_offset) &&
                        (!EXT || p.ext.window == 0 || tile0 >= q_offset + Sqc - p.ext.window);
      auto visible = [&](int r) -> bool {
        return key < hi && key <= lim_sm[r] && (!EXT || key > limlo_sm[r]);
      };
      // pass 1: per-row max over the tile's visible keys
      for (int q = 0; q < RP / 16; ++q) {
        float v[16];
        tmem_ld16(tmem + lane_off + TS(sb) + 16 * q, v);
        if (EXT)
          ext_rows16(v, xe, c2, key, t, q, slope_sm, pos_sm, mtile, mrows, q_offset, mrow_sm, hi);
        if (!full) {
#pragma unroll
          for (int e = 0; e < 16; ++e)
            if (!visible(16 * q + e)) v[e] = -INFINITY;
        }
        const float x = warp_reduce16<true>(v, lane);
        if (lane < 16) red_max[warp * RP + 16 * q + lane] = x;
      }
      named_bar_sync(1, 128);
      if (t < RP) {
        const float mt = fmaxf(fmaxf(red_max[t], red_max[RP + t]), fmaxf(red_max[2 * RP + t], red_max[3 * RP + t]));
        const float m_tile = EXT ? mt : mt * c2;
        const float m_old = m_sm[t];
        float m_new = m_old, alpha = 1.f;
        // stale-maximum threshold: 8 (log2 units) keeps p <= 2^8 for bf16 P;
        // fp8 P is stored as 64 p (p <= 4 keeps it <= 256, inside e4m3)
        if (m_tile > m_old + (FP8 ? 2.f : 8.f)) {
          m_new = m_tile;
          alpha = ex2_approx(m_old - m_new);
          *resc_flag = 1;
        }
        m_sm[t] = m_new;
        alpha_sm[t] = alpha;
        msub_sm[t] = (m_new == -INFINITY) ? 0.f : m_new - (FP8 ? 6.f : 0.f);
      }
      // P buffer sb was read by the P.V of tile j-2: wait for it before rewriting
      const bool got_pb = (j < 2) || mbar_wait(bar(BAR_PV0 + sb), (uint32_t)((j - 2) >> 1) & 1u, wd);
      if (named_bar_or(1, 128, !got_pb)) { ok = false; break; }
      tc_fence_after();
      const bool rescale = (jl > 0) && (*resc_flag != 0);
      // pass 2: exponentials, P (bf16) into the swizzled B-operand buffer
      {
        for (int q = 0; q < RP / 16; ++q) {
          float v[16];
          tmem_ld16(tmem + lane_off + TS(sb) + 16 * q, v);
          if (EXT) {
            ext_rows16(v, xe, c2, key, t, q, slope_sm, pos_sm, mtile, mrows, q_offset, mrow_sm, hi);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float4 w = reinterpret_cast<const float4*>(msub_sm + 16 * q)[i];
              v[4 * i] -= w.x; v[4 * i + 1] -= w.y; v[4 * i + 2] -= w.z; v[4 * i + 3] -= w.w;
            }
          }
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int r = 16 * q + e;
            float pv = EXT ? ex2_approx(v[e]) : ex2_approx(fmaf(v[e], c2, -msub_sm[r]));
            if (!full && !visible(r)) pv = 0.f;
            v[e] = pv;
          }
          store_p16(sb, q, v);
          const float s = warp_reduce16<false>(v, lane);
          if (lane < 16) red_sum[warp * RP + 16 * q + lane] = s;
        }
      }
      if (rescale) {
        // O^T is accumulated by the P.V of tile j-1: it must have completed
        const bool got_o = mbar_wait(bar(BAR_PV0 + (sb ^ 1)), (uint32_t)((j - 1) >> 1) & 1u, wd);
        if (named_bar_or(1, 128, !got_o)) { ok = false; break; }
        tc_fence_after();
        for (int c = 0; c < KC; ++c) {
          for (int q = 0; q < RP / 16; ++q) {
            float v[16];
            const uint32_t addr = tmem + lane_off + TO(c, cs.ob) + 16 * q;
            tmem_ld16(addr, v);
            uint32_t u[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) u[e] = __float_as_uint(v[e] * alpha_sm[16 * q + e]);
            tmem_st16(addr, u);
          }
        }
      }
      named_bar_sync(1, 128);
      if (t < RP) {
        l_sm[t] = alpha_sm[t] * l_sm[t] + (red_sum[t] + red_sum[RP + t]) + (red_sum[2 * RP + t] + red_sum[3 * RP + t]);
      }
      if (t == 0) *resc_flag = 0;
      fence_proxy_async_smem();
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(BAR_P0 + sb));
      // the pending split's last P.V is P.V(j-1) or earlier, and the wait for
      // P buffer sb above (tile j >= 2) covered P.V(j-2); flush it once that
      // covers it
      if (pend >= 0 && j >= 2 && pend_last <= j - 2) {
        write_o(pend);
        pend = -1;
      }
    }
    // no mask copy may outlive the loop (it also ends early on a give-up)
    if (EXT && p.mask_rows > 0) cp_async_wait<0>();
    // ---- the pending split and the last one ----
    if (ok && pend >= 0) {
      if (pv_done(pend_last)) write_o(pend);
      else ok = false;
    }
    if (CM && ok) {
      // the whole range is one split: leave (m, l) and v_scale * O^T (as
      // X[row][d]) in shared memory for the cluster's merge; the ring is
      // idle once the last P.V has completed
      if (pv_done(T - 1)) {
        for (int c = 0; c < KC; ++c) {
          for (int q = 0; q < RP / 16; ++q) {
            float v[16];
            tmem_ld16(tmem + lane_off + TO(c, seg_sm[0].ob) + 16 * q, v);   // warp-collective
            if (c * 128 + t < D)
#pragma unroll
              for (int e = 0; e < 16; ++e) xbuf[(size_t)(16 * q + e) * D + c * 128 + t] = v[e] * vs;
          }
        }
      } else {
        ok = false;
      }
    } else if (ok) {
      stats(seg_of(T - 1));
      if (pv_done(T - 1)) write_o(seg_of(T - 1));
      else ok = false;
    }
    tc_fence_before();
  }

  __syncwarp();
  __syncthreads();
  if (*abort_flag) {
    if (warp == WARP_PRODUCER && lane == 0) {
      drain_wait(bar(BAR_Q), 0, p.timeout_ns);
      for (int n = max(0, issued - nbuf); n < issued; ++n)
        drain_wait(bar(bar_full(n % nbuf)), (uint32_t)(n / nbuf) & 1u, p.timeout_ns);
    }
    if (warp == WARP_MMA && lane == 0) {
      mma_commit(bar(BAR_DRAIN));
      drain_wait(bar(BAR_DRAIN), 0, p.timeout_ns);
    }
    __syncwarp();
    __syncthreads();
  }
  if (warp == WARP_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, tmem_cols);
  }
  if constexpr (CM) {
    cg::this_cluster().sync();   // every CTA's (m, l) and X are in place
    if (threadIdx.x < 128) cluster_merge<DV, EXT, FP8>(p, m_sm, l_sm, xbuf, wbuf, R, RP, g, kvh, b, s0, threadIdx.x);
    cg::this_cluster().sync();   // no CTA exits while a peer reads its shared memory
  }
}

template <int DK, int DV, bool EXT, bool PAGED, bool FP8>
int launch_t(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
             const DecodeParams& p, cudaStream_t stream) {
  const Layout L(DK, p.RP, p.nbuf, p.mask_rows, FP8);
  dim3 grid((unsigned)((p.num_splits + p.group - 1) / p.group), (unsigned)(p.B * p.Hkv * p.nqc));
  cudaError_t e;
  if (p.cmerge) {
    // one cluster of num_splits CTAs per (b, kvh)
    auto kern = decode_split_kernel<DK, DV, EXT, PAGED, FP8, true>;
    const int n = p.num_splits;
    if (p.group != 1 || n < 1 || n > MAX_CLUSTER || (n & (n - 1)) != 0 || DV % n != 0) return (int)cudaErrorInvalidValue;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L.total);
    if (e != cudaSuccess) return (int)e;
    if (n > 8) {
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
      if (e != cudaSuccess) return (int)e;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = L.total;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)n;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, tq, tk, tv, p);
    if (e != cudaSuccess) return (int)e;
    return (int)cudaGetLastError();
  }
  auto kern = decode_split_kernel<DK, DV, EXT, PAGED, FP8, false>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L.total);
  if (e != cudaSuccess) return (int)e;
  kern<<<grid, THREADS, L.total, stream>>>(tq, tk, tv, p);
  return (int)cudaGetLastError();
}

template <int DK, int DV, bool FP8>
int launch_d(bool ext, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
             const DecodeParams& p, cudaStream_t stream) {
  const bool paged = p.block_table != nullptr;
  if (ext)
    return paged ? launch_t<DK, DV, true, true, FP8>(tq, tk, tv, p, stream)
                 : launch_t<DK, DV, true, false, FP8>(tq, tk, tv, p, stream);
  return paged ? launch_t<DK, DV, false, true, FP8>(tq, tk, tv, p, stream)
               : launch_t<DK, DV, false, false, FP8>(tq, tk, tv, p, stream);
}

}  // namespace

size_t decode_smem_bytes(int D, int RP, int nbuf, int mask_rows, bool fp8) {
  return Layout(D, RP, nbuf, mask_rows, fp8).total;
}

int decode_max_nbuf() { return MAX_NBUF; }

int decode_max_group() { return MAX_GROUP; }

int decode_max_cluster() { return MAX_CLUSTER; }

int launch_decode_split(int D, int Dv, bool ext, bool fp8, const CUtensorMap& tq, const CUtensorMap& tk,
                        const CUtensorMap& tv, const DecodeParams& p, cudaStream_t stream) {
  if (D == Dv) {
    switch (D) {
      case 64: return fp8 ? (int)cudaErrorInvalidValue : launch_d<64, 64, false>(ext, tq, tk, tv, p, stream);
      case 128: return fp8 ? launch_d<128, 128, true>(ext, tq, tk, tv, p, stream) : launch_d<128, 128, false>(ext, tq, tk, tv, p, stream);
      case 256: return fp8 ? launch_d<256, 256, true>(ext, tq, tk, tv, p, stream) : launch_d<256, 256, false>(ext, tq, tk, tv, p, stream);
      case 512: return fp8 ? launch_d<512, 512, true>(ext, tq, tk, tv, p, stream) : launch_d<512, 512, false>(ext, tq, tk, tv, p, stream);
      default: return (int)cudaErrorInvalidValue;
    }
  }
  // asymmetric head sizes (bf16 K/V): Q.K over D columns, V and O over Dv
  if (fp8) return (int)cudaErrorInvalidValue;
  if (D == 576 && Dv == 512) return launch_d<576, 512, false>(ext, tq, tk, tv, p, stream);
  if (D == 320 && Dv == 256) return launch_d<320, 256, false>(ext, tq, tk, tv, p, stream);
  if (D == 192 && Dv == 128) return launch_d<192, 128, false>(ext, tq, tk, tv, p, stream);
  return (int)cudaErrorInvalidValue;
}

bool decode_dims_supported(int D, int Dv, bool fp8) {
  if (D == Dv) return (D == 64 && !fp8) || D == 128 || D == 256 || D == 512;
  return !fp8 && ((D == 576 && Dv == 512) || (D == 320 && Dv == 256) || (D == 192 && Dv == 128));
}

}  // namespace gqa
