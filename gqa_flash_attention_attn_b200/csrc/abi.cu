// C ABI of the library: argument checks, TMA descriptors, launches, status.
// Every check that can fail runs on the host before any CUDA call, so bad
// arguments never reach a kernel.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "attn.h"
#include "kernels.h"

namespace gqa {
int prefill_slots(int Dv);
bool prefill_dims_supported(int D, int Dv);
int decode_max_nbuf();
}  // namespace gqa

namespace {

__device__ int g_attn_status = 0;

constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s per pipeline wait
constexpr float kLog2e = 1.4426950408889634f;
constexpr size_t kTwoCtaSmemLimit = 115712;  // two CTAs per SM
constexpr size_t kOneCtaSmemLimit = 232448;  // the most one CTA may have
constexpr int kMaxFusedCluster = 8;          // CTAs per cluster in attn_decode_fused

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

std::mutex g_mu;
EncodeTiledFn g_encode = nullptr;
int* g_status_ptr[64] = {nullptr};

int cuda_fail() { return ATTN_ERR_CUDA; }

EncodeTiledFn encoder() {
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_encode == nullptr) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  }
  return g_encode;
}

int sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  static int cached[64] = {0};
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    cached[dev] = n;
  }
  return cached[dev];
}

int* status_ptr() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_status_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_attn_status) != cudaSuccess) return nullptr;
    g_status_ptr[dev] = static_cast<int*>(p);
  }
  return g_status_ptr[dev];
}

// Tensor with dimensions d0 (innermost, contiguous) .. d3 and element strides
// s1..s3 of the outer three, tiled with 128-byte swizzle; bf16, or one-byte
// codes when fp8.
bool make_map_strided(CUtensorMap* m, const void* ptr, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t d3,
                      uint64_t s1, uint64_t s2, uint64_t s3, uint32_t b0, uint32_t b1, uint32_t b2, uint32_t b3,
                      bool fp8 = false) {
  EncodeTiledFn enc = encoder();
  if (enc == nullptr) return false;
  const uint64_t eb = fp8 ? 1 : 2;
  const cuuint64_t dims[4] = {d0, d1, d2, d3};
  const cuuint64_t strides[3] = {s1 * eb, s2 * eb, s3 * eb};
  const cuuint32_t box[4] = {b0, b1, b2, b3};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  std::memset(m, 0, sizeof(*m));
  return enc(m, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Contiguous bf16 tensor [d3][d2][d1][d0].
bool make_map(CUtensorMap* m, const void* ptr, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t d3, uint32_t b0,
              uint32_t b1, uint32_t b2, uint32_t b3) {
  return make_map_strided(m, ptr, d0, d1, d2, d3, d0, d0 * d1, d0 * d1 * d2, b0, b1, b2, b3);
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// Shape checks shared by prefill and decode.
int check_common(const void* q, const void* k, const void* v, int B, int Hq, int Hkv, int Sq, int Skv, int D,
                 int q_offset, int causal, float scale) {
  if (q == nullptr || k == nullptr || v == nullptr) return ATTN_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || Sq < 1 || Skv < 1 || D < 1) return ATTN_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return ATTN_ERR_INVALID_ARG;
  if (q_offset < 0 || (long long)q_offset + Sq > 0x7fffffffLL) return ATTN_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return ATTN_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
  // TMA strides must stay below 2^40 bytes
  if ((long double)B * Sq * Hq * D * 4 >= 1099511627776.0L) return ATTN_ERR_INVALID_ARG;
  if ((long double)B * Skv * Hkv * D * 2 >= 1099511627776.0L) return ATTN_ERR_INVALID_ARG;
  return ATTN_OK;
}

// Validates *opt and fills the kernels' form of it.  *on is false when every
// term is off, so the plain kernels run.
int make_ext(const attn_options* opt, int Hq, int Sq, int Skv, int q_offset, int causal, float scale,
             bool allow_sinks, gqa::LogitExt* ext, bool* on) {
  *ext = gqa::LogitExt{};
  *on = false;
  if (opt == nullptr) return ATTN_OK;
  if (!std::isfinite(opt->softcap) || opt->softcap < 0.f) return ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(opt->alibi_max_bias) || opt->alibi_max_bias < 0.f) return ATTN_ERR_INVALID_ARG;
  if (opt->window < 0) return ATTN_ERR_INVALID_ARG;
  if (opt->sinks != nullptr && !allow_sinks) return ATTN_ERR_INVALID_ARG;
  if (opt->sinks != nullptr && !aligned(opt->sinks, 4)) return ATTN_ERR_ALIGNMENT;
  if (opt->window > 0 && (causal != 1 || (long long)q_offset + Sq > Skv)) return ATTN_ERR_UNSUPPORTED;
  if (opt->softcap > 0.f) {
    ext->cap_a = scale / opt->softcap;
    ext->cap_b = opt->softcap * kLog2e;
    if (!(ext->cap_a > 0.f) || !std::isfinite(ext->cap_a)) return ATTN_ERR_INVALID_ARG;
  }
  if (opt->alibi_max_bias > 0.f) {
    int n2 = 1;
    while (2 * n2 <= Hq) n2 *= 2;
    ext->alibi = 1;
    ext->n2 = n2;
    ext->l2m0 = -opt->alibi_max_bias / (float)n2;
    ext->l2m1 = -opt->alibi_max_bias / (float)(2 * n2);
  }
  if (opt->mask != nullptr) {
    if (opt->mask_stride_seq < 0 || opt->mask_stride_row < 0) return ATTN_ERR_INVALID_ARG;
    if (!aligned(opt->mask, 2)) return ATTN_ERR_ALIGNMENT;
    ext->mask = static_cast<const uint16_t*>(opt->mask);
    ext->mask_sb = opt->mask_stride_seq;
    ext->mask_sr = opt->mask_stride_row;
  }
  ext->sinks = opt->sinks;
  ext->window = opt->window;
  *on = ext->cap_a > 0.f || ext->alibi != 0 || ext->sinks != nullptr || ext->window > 0 || ext->mask != nullptr;
  return ATTN_OK;
}

// Checks of a K/V view before any CUDA call: strides, paging, element type.
// *fp8 tells the element type.
int check_view(const attn_kv_view* kv, int Skv, bool* fp8) {
  const bool own_v = kv->v_stride_seq != 0 || kv->v_stride_token != 0 || kv->v_stride_head != 0;
  const long long strides[6] = {kv->stride_head,  kv->stride_token, kv->stride_seq,
                                own_v ? kv->v_stride_head : kv->stride_head,
                                own_v ? kv->v_stride_token : kv->stride_token,
                                own_v ? kv->v_stride_seq : kv->stride_seq};
  for (long long x : strides)
    if (x < 1 || x >= (1LL << 37)) return ATTN_ERR_INVALID_ARG;
  if (kv->block_table != nullptr) {
    const int ps = kv->page_size;
    if (!(ps == 16 || ps == 32 || ps == 64 || (ps >= 128 && ps % 128 == 0))) return ATTN_ERR_INVALID_ARG;
    if (kv->max_pages < 1 || kv->num_pages < 1) return ATTN_ERR_INVALID_ARG;
    if ((long long)kv->max_pages * ps != Skv) return ATTN_ERR_INVALID_ARG;
    if (!aligned(kv->block_table, 4)) return ATTN_ERR_ALIGNMENT;
  }
  if (kv->seq_lens != nullptr && !aligned(kv->seq_lens, 4)) return ATTN_ERR_ALIGNMENT;
  if (kv->kv_dtype != ATTN_BF16 && kv->kv_dtype != ATTN_FP8_E4M3) return ATTN_ERR_INVALID_ARG;
  *fp8 = kv->kv_dtype == ATTN_FP8_E4M3;
  if (*fp8 && (kv->k_scale == nullptr || kv->v_scale == nullptr || !aligned(kv->k_scale, 4) ||
               !aligned(kv->v_scale, 4)))
    return ATTN_ERR_INVALID_ARG;
  if (kv->head_dim_v < 0) return ATTN_ERR_INVALID_ARG;
  if (kv->k == nullptr || kv->v == nullptr) return ATTN_ERR_INVALID_ARG;
  if (!aligned(kv->k, 16) || !aligned(kv->v, 16)) return ATTN_ERR_ALIGNMENT;
  for (long long x : strides)
    if (x % (*fp8 ? 16 : 8) != 0) return ATTN_ERR_ALIGNMENT;
  return ATTN_OK;
}

struct ViewStrides {
  uint64_t head, token, seq;
};
ViewStrides k_strides(const attn_kv_view* kv) {
  return {(uint64_t)kv->stride_head, (uint64_t)kv->stride_token, (uint64_t)kv->stride_seq};
}
// V's strides: its own when any is set, else K's
ViewStrides v_strides(const attn_kv_view* kv) {
  if (kv->v_stride_seq != 0 || kv->v_stride_token != 0 || kv->v_stride_head != 0)
    return {(uint64_t)kv->v_stride_head, (uint64_t)kv->v_stride_token, (uint64_t)kv->v_stride_seq};
  return k_strides(kv);
}

// Tensor maps of a K/V view for the split-KV kernel: K (D columns) and V (Dv
// columns) over (d, kvh, key, sequence), or (d, kvh, row in page, page).
bool view_maps(const attn_kv_view* kv, int D, int Dv, int Hkv, int Skv, int B, bool fp8, CUtensorMap* tk,
               CUtensorMap* tv) {
  const bool paged = kv->block_table != nullptr;
  const uint64_t d2 = paged ? (uint64_t)kv->page_size : (uint64_t)Skv;
  const uint64_t d3 = paged ? (uint64_t)kv->num_pages : (uint64_t)B;
  const uint32_t rows = paged && kv->page_size < 128 ? (uint32_t)kv->page_size : 128u;
  const uint32_t b0 = fp8 ? 128u : 64u;   // 128-byte box rows either way
  const ViewStrides k = k_strides(kv), v = v_strides(kv);
  return make_map_strided(tk, kv->k, D, Hkv, d2, d3, k.head, k.token, k.seq, b0, 1, rows, 1, fp8) &&
         make_map_strided(tv, kv->v, Dv, Hkv, d2, d3, v.head, v.token, v.seq, b0, 1, rows, 1, fp8);
}

// The view's fields in the split-KV kernel's parameters.
void view_params(const attn_kv_view* kv, bool fp8, gqa::DecodeParams& p) {
  const bool paged = kv->block_table != nullptr;
  const ViewStrides ks = k_strides(kv), vs = v_strides(kv);
  p.kv_shared = kv->v == kv->k && ks.head == vs.head && ks.token == vs.token && ks.seq == vs.seq;
  p.seq_lens = kv->seq_lens;
  p.block_table = kv->block_table;
  p.max_pages = paged ? kv->max_pages : 0;
  p.page_size = paged ? kv->page_size : 0;
  p.k_scale = fp8 ? kv->k_scale : nullptr;
  p.v_scale = fp8 ? kv->v_scale : nullptr;
}

// Prefill through the split-KV kernel (D = 512, asymmetric head sizes,
// paged or fp8 K/V, lengths per sequence): one split, query rows cut into
// chunks of 80 / g positions per CTA, writing the final O and LSE directly.
// 80 rows fill TMEM (2 S^T buffers + O^T: 6 x 80 of 512 columns at Dv = 512),
// so a CTA takes a whole SM (its shared memory is sized past half of it);
// every K/V tile a CTA streams from L2 then serves up to 80 query rows.
int prefill_wide(const void* q, const attn_kv_view* kv, bool fp8, void* out, float* lse, int B, int Hq, int Hkv,
                 int Sq, int Skv, int D, int Dv, int q_offset, int causal, float scale, int out_dtype,
                 const gqa::LogitExt& ext, bool ext_on, void* stream) {
  const int g = Hq / Hkv;
  if (g > 32) return ATTN_ERR_UNSUPPORTED;
  if (!gqa::decode_dims_supported(D, Dv, fp8)) return ATTN_ERR_UNSUPPORTED;
  // rows per CTA: TMEM holds 2 S^T buffers and O^T, (2 + ceil(Dv/128)) x RP of 512 columns
  const int max_rows = std::min(128, (512 / (2 + (Dv + 127) / 128)) / 16 * 16);
  int qchunk = std::max(1, std::min(max_rows / g, Sq));
  // fewer rows when two K/V slots and the Q, P buffers of that many rows do
  // not fit one CTA's shared memory (fp8 at D = 512: two more Q planes)
  auto mrows_of = [&](int qc) {
    return (ext.mask != nullptr && qc <= 32 && aligned(ext.mask, 16) && ext.mask_sb % 8 == 0 &&
            ext.mask_sr % 8 == 0)
               ? qc
               : 0;
  };
  auto rp_of = [&](int qc) { return (g * qc + 15) / 16 * 16; };
  while (qchunk > 1 && gqa::decode_smem_bytes(D, rp_of(qchunk), 2, mrows_of(qchunk), fp8) > kOneCtaSmemLimit)
    --qchunk;
  const int nqc = (Sq + qchunk - 1) / qchunk;
  if ((long long)B * Hkv * nqc > 65535) return ATTN_ERR_UNSUPPORTED;   // grid rows
  gqa::DecodeParams p{};
  p.part_out = nullptr;
  p.part_lse = lse;
  p.fout = out;
  p.fout_bf16 = out_dtype == ATTN_BF16;
  p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.Sq = Sq; p.Skv = Skv;
  p.q_offset = q_offset; p.causal = causal;
  p.g = g; p.R = g * qchunk; p.RP = (p.R + 15) / 16 * 16;
  p.qchunk = qchunk;
  p.nqc = nqc;
  p.num_splits = 1;
  p.chunk = Skv;
  p.group = 1;
  p.obuf = 1;
  p.mask_rows = mrows_of(qchunk);
  // one CTA per SM: at least half of the shared memory, at most what fits
  int nbuf = 2;
  while (nbuf < gqa::decode_max_nbuf() &&
         gqa::decode_smem_bytes(D, p.RP, nbuf + 1, p.mask_rows, fp8) <= kOneCtaSmemLimit)
    ++nbuf;
  if (gqa::decode_smem_bytes(D, p.RP, nbuf, p.mask_rows, fp8) > kOneCtaSmemLimit) return ATTN_ERR_UNSUPPORTED;
  p.nbuf = nbuf;
  p.c2 = scale * kLog2e;
  p.timeout_ns = kWaitLimitNs;
  p.ext = ext;
  view_params(kv, fp8, p);
  p.status = status_ptr();
  if (p.status == nullptr) return cuda_fail();
  CUtensorMap tq, tk, tv;
  if (!make_map(&tq, q, D, Hq, Sq, B, 64, (uint32_t)g, (uint32_t)qchunk, 1)) return cuda_fail();
  if (!view_maps(kv, D, Dv, Hkv, Skv, B, fp8, &tk, &tv)) return cuda_fail();
  return gqa::launch_decode_split(D, Dv, ext_on, fp8, tq, tk, tv, p, static_cast<cudaStream_t>(stream)) == 0
             ? ATTN_OK
             : ATTN_ERR_CUDA;
}

// The prefill kernel over given K/V tensor maps (D = Dv in 64, 128, 256, or
// D = 192 with Dv = 128).  tk64 (K in 64-key boxes, or nullptr) enables the
// CTA-pair form at D = Dv = 256 with an even group size and no mask.
int prefill_fast(const void* q, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap* tk64, void* out,
                 float* lse, int B, int Hq, int Hkv, int Sq, int Skv, int D, int Dv, int q_offset, int causal,
                 float scale, int out_dtype, const gqa::LogitExt& ext, bool ext_on, void* stream) {
  const int nslot = gqa::prefill_slots(Dv);
  const int g = Hq / Hkv;
  const bool pair = tk64 != nullptr && D == 256 && Dv == 256 && g % 2 == 0 && ext.mask == nullptr;
  gqa::PrefillParams p{};
  p.out = out;
  p.lse = lse;
  p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.Sq = Sq; p.Skv = Skv;
  p.q_offset = q_offset; p.causal = causal; p.out_f32 = (out_dtype == ATTN_F32);
  p.g = g;
  p.units_per_kvh = pair ? g / 2 : (g + nslot - 1) / nslot;
  p.n_qt = (Sq + 127) / 128;
  p.c2 = scale * kLog2e;
  p.timeout_ns = kWaitLimitNs;
  p.ext = ext;
  if ((long long)p.n_qt * B * Hkv * p.units_per_kvh > 0x7fffffffLL) return ATTN_ERR_INVALID_ARG;

  p.status = status_ptr();
  if (p.status == nullptr) return cuda_fail();
  p.num_ctas = sm_count();
  if (p.num_ctas <= 0) return cuda_fail();
  CUtensorMap tq;
  if (!make_map(&tq, q, D, Hq, Sq, B, 64, 1, 128, 1)) return cuda_fail();
  if (pair)
    return gqa::launch_prefill_pair(D, ext_on, tq, *tk64, tv, p, static_cast<cudaStream_t>(stream)) == 0
               ? ATTN_OK
               : ATTN_ERR_CUDA;
  // the additive mask staged by TMA: 16-byte aligned rows, and every head
  // slot of a CTA visits every tile (one slot, or an even group size)
  CUtensorMap tm;
  std::memset(&tm, 0, sizeof(tm));
  if (ext.mask != nullptr && aligned(ext.mask, 16) && ext.mask_sr % 8 == 0 && ext.mask_sb % 8 == 0 &&
      ext.mask_sr > 0 && (nslot == 1 || g % 2 == 0)) {
    const uint64_t bm = ext.mask_sb != 0 ? (uint64_t)B : 1u;
    const uint64_t s2 = ext.mask_sb != 0 ? (uint64_t)ext.mask_sb : (uint64_t)Sq * ext.mask_sr;
    if (!make_map_strided(&tm, ext.mask, Skv, Sq, bm, 1, (uint64_t)ext.mask_sr, s2, s2 * bm, 64, 128, 1, 1))
      return cuda_fail();
    p.mask_tma = 1;
  }
  return gqa::launch_prefill(D, Dv, ext_on, tq, tk, tv, tm, p, static_cast<cudaStream_t>(stream)) == 0
             ? ATTN_OK
             : ATTN_ERR_CUDA;
}

// The contiguous [B, Skv, Hkv, D] view of k and v.
attn_kv_view contiguous_view(const void* k, const void* v, int Skv, int Hkv, int D) {
  attn_kv_view kv{};
  kv.k = k;
  kv.v = v;
  kv.stride_head = D;
  kv.stride_token = (long long)Hkv * D;
  kv.stride_seq = (long long)Skv * Hkv * D;
  return kv;
}

// Split-KV decode over a view: partials (fused = false), or one launch whose
// clusters merge the key ranges and write the final O and LSE (fused).
int decode_run(const void* q, const attn_kv_view* kv, float* partial_out, float* partial_lse, void* out,
               float* lse, int out_dtype, bool fused, int B, int Hq, int Hkv, int Sq, int Skv, int D, int q_offset,
               int causal, float scale, int num_splits, const attn_options* opt, void* stream) {
  if (kv == nullptr) return ATTN_ERR_INVALID_ARG;
  // with per-sequence lengths q_offset is ignored (rows sit at len_b - Sq + s)
  if (kv->seq_lens != nullptr) q_offset = 0;
  int st = check_common(q, kv->k, kv->v, B, Hq, Hkv, Sq, Skv, D, q_offset, causal, scale);
  if (st != ATTN_OK) return st;
  gqa::LogitExt ext;
  bool ext_on;
  st = make_ext(opt, Hq, Sq, Skv, q_offset, causal, scale, fused, &ext, &ext_on);
  if (st != ATTN_OK) return st;
  if (fused) {
    if (out == nullptr) return ATTN_ERR_INVALID_ARG;
    if (out_dtype != ATTN_BF16 && out_dtype != ATTN_F32) return ATTN_ERR_INVALID_ARG;
  } else if (partial_out == nullptr || partial_lse == nullptr) {
    return ATTN_ERR_INVALID_ARG;
  }
  if (num_splits < 1 || num_splits > Skv || num_splits > 65535) return ATTN_ERR_INVALID_ARG;
  bool fp8 = false;
  st = check_view(kv, Skv, &fp8);
  if (st != ATTN_OK) return st;
  const int Dv = kv->head_dim_v != 0 ? kv->head_dim_v : D;
  if (!gqa::decode_dims_supported(D, Dv, fp8)) return ATTN_ERR_UNSUPPORTED;
  const int g = Hq / Hkv;
  const long long R = (long long)g * Sq;
  const long long RP = (R + 15) / 16 * 16;
  const int vchunks = (Dv + 127) / 128;   // O^T chunks of 128 d-rows (one at Dv = 64)
  if (RP * (2 + vchunks) > 256) return ATTN_ERR_UNSUPPORTED;  // TMEM: two S^T buffers + O^T
  if (g > 256 || Sq > 256) return ATTN_ERR_UNSUPPORTED;  // TMA box extents
  if ((long long)B * Hkv > 65535) return ATTN_ERR_INVALID_ARG;
  if (!aligned(q, 16)) return ATTN_ERR_ALIGNMENT;
  if (fused) {
    if (!aligned(out, 16) || (lse != nullptr && !aligned(lse, 4))) return ATTN_ERR_ALIGNMENT;
  } else if (!aligned(partial_out, 16) || !aligned(partial_lse, 4)) {
    return ATTN_ERR_ALIGNMENT;
  }
  // fused: key ranges per (b, kvh) = the cluster size, the largest power of
  // two <= min(num_splits, 8).  Clusters of 16 ran slower in every measured
  // shape (D512 decode 145 vs 117 us, verify 182 vs 111 us): fewer of them
  // are resident at once than their CTA count suggests.
  int nsplit = num_splits;
  if (fused) {
    nsplit = 1;
    while (nsplit * 2 <= std::min(num_splits, kMaxFusedCluster)) nsplit *= 2;
  }

  gqa::DecodeParams p{};
  p.part_out = fused ? nullptr : partial_out;
  p.part_lse = fused ? lse : partial_lse;
  p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.Sq = Sq; p.Skv = Skv;
  p.q_offset = q_offset; p.causal = causal;
  p.g = g; p.R = (int)R; p.RP = (int)RP;
  p.num_splits = nsplit;
  p.chunk = (Skv + nsplit - 1) / nsplit;
  // stage the additive mask per tile in shared memory (cp.async, 16-byte
  // chunks) for up to 32 query rows when its rows are 16-byte aligned
  p.mask_rows = (ext.mask != nullptr && Sq <= 32 && aligned(ext.mask, 16) && ext.mask_sb % 8 == 0 &&
                 ext.mask_sr % 8 == 0)
                    ? Sq
                    : 0;
  // ring slots: as many as keep two CTAs per SM, or, when even two slots
  // leave room for one CTA only, as many as that CTA can hold
  const size_t smem_limit =
      gqa::decode_smem_bytes(D, p.RP, 2, p.mask_rows, fp8) <= kTwoCtaSmemLimit ? kTwoCtaSmemLimit : kOneCtaSmemLimit;
  int nbuf = 2;
  while (nbuf < gqa::decode_max_nbuf() && gqa::decode_smem_bytes(D, p.RP, nbuf + 1, p.mask_rows, fp8) <= smem_limit)
    ++nbuf;
  if (gqa::decode_smem_bytes(D, p.RP, nbuf, p.mask_rows, fp8) > kOneCtaSmemLimit) return ATTN_ERR_UNSUPPORTED;
  p.nbuf = nbuf;
  if (fused) {
    // the merge's shared memory (X [RP][Dv] fp32, weights [16][RP], 1/L [RP])
    // reuses the idle K/V ring
    const long long need = RP * Dv * 4 + (long long)(gqa::decode_max_cluster() + 1) * RP * 4;
    if (need > (long long)nbuf * (fp8 ? 16384 : 32768)) return ATTN_ERR_UNSUPPORTED;
    p.group = 1;
    p.obuf = 1;
    p.cmerge = 1;
    p.fout = out;
    p.fout_bf16 = out_dtype == ATTN_BF16;
  } else {
    // Consecutive splits per CTA: enough that the CTAs fit the resident slots
    // (two per SM when the shared memory allows) in one wave, at most 8.
    const int nsm = sm_count();
    if (nsm <= 0) return cuda_fail();
    const long long slots =
        (long long)nsm * (gqa::decode_smem_bytes(D, p.RP, nbuf, p.mask_rows, fp8) <= kTwoCtaSmemLimit ? 2 : 1);
    const long long units = (long long)num_splits * B * Hkv;
    long long grp = (units + slots - 1) / slots;
    grp = std::min<long long>(std::min<long long>(grp, gqa::decode_max_group()), num_splits);
    p.group = (int)std::max<long long>(grp, 1);
    // two O^T buffers when split boundaries exist and two CTAs' TMEM still fits
    p.obuf = (p.group > 1 && RP * (2 + 2 * vchunks) <= 256) ? 2 : 1;
    p.fout = nullptr;
  }
  p.c2 = scale * kLog2e;
  p.timeout_ns = kWaitLimitNs;
  p.ext = ext;
  view_params(kv, fp8, p);
  p.qchunk = Sq;
  p.nqc = 1;

  p.status = status_ptr();
  if (p.status == nullptr) return cuda_fail();
  CUtensorMap tq, tk, tv;
  if (!make_map(&tq, q, D, Hq, Sq, B, 64, (uint32_t)g, (uint32_t)Sq, 1)) return cuda_fail();
  if (!view_maps(kv, D, Dv, Hkv, Skv, B, fp8, &tk, &tv)) return cuda_fail();
  const cudaStream_t st_ = static_cast<cudaStream_t>(stream);
  return gqa::launch_decode_split(D, Dv, ext_on, fp8, tq, tk, tv, p, st_) == 0 ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // namespace

extern "C" {

int attn_version(void) { return 0x000500; }

const char* attn_status_string(int status) {
  switch (status) {
    case ATTN_OK: return "ok";
    case ATTN_ERR_INVALID_ARG: return "invalid argument";
    case ATTN_ERR_UNSUPPORTED: return "unsupported shape";
    case ATTN_ERR_ALIGNMENT: return "misaligned pointer";
    case ATTN_ERR_CUDA: return "CUDA error";
    case ATTN_ERR_TIMEOUT: return "pipeline wait timed out";
    case ATTN_ERR_TOO_LARGE: return "problem exceeds the fixed no-alloc scratch";
    default: return "unknown status";
  }
}

int attn_prefill(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Hq, int Hkv,
                 int Sq, int Skv, int D, int q_offset, int causal, float scale, int out_dtype, void* stream) {
  return attn_prefill_ex(q, k, v, out, lse, B, Hq, Hkv, Sq, Skv, D, q_offset, causal, scale, out_dtype, nullptr,
                         stream);
}

int attn_prefill_ex(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Hq, int Hkv,
                    int Sq, int Skv, int D, int q_offset, int causal, float scale, int out_dtype,
                    const attn_options* opt, void* stream) {
  int st = check_common(q, k, v, B, Hq, Hkv, Sq, Skv, D, q_offset, causal, scale);
  if (st != ATTN_OK) return st;
  gqa::LogitExt ext;
  bool ext_on;
  st = make_ext(opt, Hq, Sq, Skv, q_offset, causal, scale, true, &ext, &ext_on);
  if (st != ATTN_OK) return st;
  if (out == nullptr) return ATTN_ERR_INVALID_ARG;
  if (out_dtype != ATTN_BF16 && out_dtype != ATTN_F32) return ATTN_ERR_INVALID_ARG;
  if (D != 64 && D != 128 && D != 256 && D != 512) return ATTN_ERR_UNSUPPORTED;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16)) return ATTN_ERR_ALIGNMENT;
  if (lse != nullptr && !aligned(lse, 4)) return ATTN_ERR_ALIGNMENT;
  if (D == 512) {
    const attn_kv_view kv = contiguous_view(k, v, Skv, Hkv, D);
    return prefill_wide(q, &kv, false, out, lse, B, Hq, Hkv, Sq, Skv, D, D, q_offset, causal, scale, out_dtype, ext,
                        ext_on, stream);
  }
  CUtensorMap tk, tv, tk64;
  if (!make_map(&tk, k, D, Hkv, Skv, B, 64, 1, 128, 1)) return cuda_fail();
  if (!make_map(&tv, v, D, Hkv, Skv, B, 64, 1, 128, 1)) return cuda_fail();
  const bool k64 = D == 256;   // K in 64-key boxes for the CTA-pair form
  if (k64 && !make_map(&tk64, k, D, Hkv, Skv, B, 64, 1, 64, 1)) return cuda_fail();
  return prefill_fast(q, tk, tv, k64 ? &tk64 : nullptr, out, lse, B, Hq, Hkv, Sq, Skv, D, D, q_offset, causal, scale,
                      out_dtype, ext, ext_on, stream);
}

int attn_prefill_kv(const void* q, const attn_kv_view* kv, void* out, float* lse, int B, int Hq, int Hkv, int Sq,
                    int Skv, int D, int q_offset, int causal, float scale, int out_dtype, const attn_options* opt,
                    void* stream) {
  if (kv == nullptr) return ATTN_ERR_INVALID_ARG;
  if (kv->seq_lens != nullptr) q_offset = 0;   // rows sit at len_b - Sq + s
  int st = check_common(q, kv->k, kv->v, B, Hq, Hkv, Sq, Skv, D, q_offset, causal, scale);
  if (st != ATTN_OK) return st;
  gqa::LogitExt ext;
  bool ext_on;
  st = make_ext(opt, Hq, Sq, Skv, q_offset, causal, scale, true, &ext, &ext_on);
  if (st != ATTN_OK) return st;
  if (out == nullptr) return ATTN_ERR_INVALID_ARG;
  if (out_dtype != ATTN_BF16 && out_dtype != ATTN_F32) return ATTN_ERR_INVALID_ARG;
  bool fp8 = false;
  st = check_view(kv, Skv, &fp8);
  if (st != ATTN_OK) return st;
  const int Dv = kv->head_dim_v != 0 ? kv->head_dim_v : D;
  const bool fast = gqa::prefill_dims_supported(D, Dv) && !fp8 && kv->block_table == nullptr &&
                    kv->seq_lens == nullptr;
  if (!fast && !gqa::decode_dims_supported(D, Dv, fp8)) return ATTN_ERR_UNSUPPORTED;
  if (!aligned(q, 16) || !aligned(out, 16)) return ATTN_ERR_ALIGNMENT;
  if (lse != nullptr && !aligned(lse, 4)) return ATTN_ERR_ALIGNMENT;
  if (!fast)
    return prefill_wide(q, kv, fp8, out, lse, B, Hq, Hkv, Sq, Skv, D, Dv, q_offset, causal, scale, out_dtype, ext,
                        ext_on, stream);
  CUtensorMap tk, tv, tk64;
  const ViewStrides ks = k_strides(kv), vs = v_strides(kv);
  if (!make_map_strided(&tk, kv->k, D, Hkv, Skv, B, ks.head, ks.token, ks.seq, 64, 1, 128, 1)) return cuda_fail();
  if (!make_map_strided(&tv, kv->v, Dv, Hkv, Skv, B, vs.head, vs.token, vs.seq, 64, 1, 128, 1)) return cuda_fail();
  const bool k64 = D == 256 && Dv == 256;   // K in 64-key boxes for the CTA-pair form
  if (k64 && !make_map_strided(&tk64, kv->k, D, Hkv, Skv, B, ks.head, ks.token, ks.seq, 64, 1, 64, 1))
    return cuda_fail();
  return prefill_fast(q, tk, tv, k64 ? &tk64 : nullptr, out, lse, B, Hq, Hkv, Sq, Skv, D, Dv, q_offset, causal, scale,
                      out_dtype, ext, ext_on, stream);
}

size_t attn_decode_workspace_bytes(int B, int Hq, int Sq, int D, int num_splits) {
  if (B < 1 || Hq < 1 || Sq < 1 || D < 1 || num_splits < 1) return 0;
  const size_t n_out = (size_t)num_splits * B * Sq * Hq * D;
  const size_t n_lse = (size_t)num_splits * B * Hq * Sq;
  return (n_out + n_lse) * sizeof(float);
}

int attn_decode_split(const void* q, const void* k, const void* v, float* partial_out, float* partial_lse,
                      int B, int Hq, int Hkv, int Sq, int Skv, int D, int q_offset, int causal, float scale,
                      int num_splits, void* stream) {
  return attn_decode_split_ex(q, k, v, partial_out, partial_lse, B, Hq, Hkv, Sq, Skv, D, q_offset, causal, scale,
                              num_splits, nullptr, stream);
}

int attn_decode_split_ex(const void* q, const void* k, const void* v, float* partial_out, float* partial_lse,
                         int B, int Hq, int Hkv, int Sq, int Skv, int D, int q_offset, int causal, float scale,
                         int num_splits, const attn_options* opt, void* stream) {
  const attn_kv_view kv = contiguous_view(k, v, Skv, Hkv, D);
  return attn_decode_split_kv(q, &kv, partial_out, partial_lse, B, Hq, Hkv, Sq, Skv, D, q_offset, causal, scale,
                              num_splits, opt, stream);
}

int attn_decode_split_kv(const void* q, const attn_kv_view* kv, float* partial_out, float* partial_lse, int B,
                         int Hq, int Hkv, int Sq, int Skv, int D, int q_offset, int causal, float scale,
                         int num_splits, const attn_options* opt, void* stream) {
  return decode_run(q, kv, partial_out, partial_lse, nullptr, nullptr, ATTN_BF16, false, B, Hq, Hkv, Sq, Skv, D,
                    q_offset, causal, scale, num_splits, opt, stream);
}

int attn_decode_fused(const void* q, const attn_kv_view* kv, void* out, float* lse, int B, int Hq, int Hkv, int Sq,
                      int Skv, int D, int q_offset, int causal, float scale, int num_splits, int out_dtype,
                      const attn_options* opt, void* stream) {
  return decode_run(q, kv, nullptr, nullptr, out, lse, out_dtype, true, B, Hq, Hkv, Sq, Skv, D, q_offset, causal,
                    scale, num_splits, opt, stream);
}

int attn_merge(const float* partial_out, const float* partial_lse, void* out, float* lse, int B, int Hq, int Sq,
               int D, int num_splits, int out_dtype, void* stream) {
  return attn_merge_ex(partial_out, partial_lse, out, lse, B, Hq, Sq, D, num_splits, out_dtype, nullptr, stream);
}

int attn_merge_ex(const float* partial_out, const float* partial_lse, void* out, float* lse, int B, int Hq,
                  int Sq, int D, int num_splits, int out_dtype, const float* sinks, void* stream) {
  if (partial_out == nullptr || partial_lse == nullptr || out == nullptr) return ATTN_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Sq < 1 || num_splits < 1) return ATTN_ERR_INVALID_ARG;
  if (out_dtype != ATTN_BF16 && out_dtype != ATTN_F32) return ATTN_ERR_INVALID_ARG;
  if (D < 4 || D > 1024 || D % 4 != 0) return ATTN_ERR_UNSUPPORTED;
  if (!aligned(partial_out, 16) || !aligned(out, out_dtype == ATTN_F32 ? 16 : 8)) return ATTN_ERR_ALIGNMENT;
  if (!aligned(partial_lse, 4) || (lse != nullptr && !aligned(lse, 4))) return ATTN_ERR_ALIGNMENT;
  if (sinks != nullptr && !aligned(sinks, 4)) return ATTN_ERR_ALIGNMENT;
  gqa::MergeParams p{};
  p.sinks = sinks;
  p.part_out = partial_out;
  p.part_lse = partial_lse;
  p.out = out;
  p.lse = lse;
  p.B = B; p.Hq = Hq; p.Sq = Sq; p.D = D; p.num_splits = num_splits;
  p.out_f32 = (out_dtype == ATTN_F32);
  return gqa::launch_merge(p, static_cast<cudaStream_t>(stream)) == 0 ? ATTN_OK : ATTN_ERR_CUDA;
}

int attn_last_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return ATTN_ERR_CUDA;
  int* sp = status_ptr();
  if (sp == nullptr) return ATTN_ERR_CUDA;
  int st = 0;
  if (cudaMemcpy(&st, sp, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return ATTN_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpy(sp, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return ATTN_ERR_CUDA;
  return st;
}

int attn_watchdog_selftest(unsigned long long limit_ns, void* stream) {
  if (limit_ns < 1000ull) limit_ns = 1000ull;
  if (limit_ns > 5000000000ull) limit_ns = 5000000000ull;
  int* sp = status_ptr();
  if (sp == nullptr) return ATTN_ERR_CUDA;
  return gqa::launch_watchdog_selftest(sp, limit_ns, static_cast<cudaStream_t>(stream)) == 0 ? ATTN_OK
                                                                                              : ATTN_ERR_CUDA;
}

}  // extern "C"
