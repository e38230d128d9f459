// Internal interface between the C-ABI layer (abi.cu) and the kernels.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace gqa {

// Optional logit terms, prepared on the host.  The logit in log2 units is
//   L = (cap_a > 0 ? cap_b * tanh(s * cap_a) : s * c2) + slope_h * log2(e) * (t - pos)
// with s the raw Q.K dot product; slope_h = 2^(l2m0 * (h + 1)) for h < n2,
// else 2^(l2m1 * (2 (h - n2) + 1)), and 0 when alibi is off; plus
// log2(e) * mask[b, s, t] when a mask is given.
struct LogitExt {
  float cap_a;        // scale / softcap, or 0 when off
  float cap_b;        // softcap * log2(e)
  int alibi;          // 0: off
  float l2m0, l2m1;   // log2 of the two ALiBi slope bases
  int n2;             // largest power of two <= Hq
  const float* sinks; // [Hq] natural-log sink logits, or nullptr
  int window;         // 0: off
  const uint16_t* mask;        // bf16 bits of the additive mask, or nullptr
  long long mask_sb, mask_sr;  // element strides: sequence, query row
};

struct PrefillParams {
  void* out;          // [B, Sq, Hq, Dv] bf16 or f32
  float* lse;         // [B, Hq, Sq] or nullptr
  int* status;        // device status word
  int B, Hq, Hkv, Sq, Skv, q_offset, causal, out_f32;
  int g;              // Hq / Hkv
  int units_per_kvh;  // head slots per K/V head: ceil(g / NSLOT)
  int n_qt;           // ceil(Sq / 128)
  int num_ctas;       // persistent grid size (SM count)
  float c2;           // scale * log2(e)
  unsigned long long timeout_ns;
  LogitExt ext;
  int mask_tma;       // the mask is staged by TMA (its map is the kernel's tm_m)
};

struct DecodeParams {
  float* part_out;    // [S, B, Sq, Hq, D]
  float* part_lse;    // [S, B, Hq, Sq]
  int* status;
  int B, Hq, Hkv, Sq, Skv, q_offset, causal;
  int g, R, RP;       // rows per K/V head = g*Sq, padded to a multiple of 16
  int num_splits, chunk;  // keys per split
  int group;              // consecutive splits per CTA (1..8), one tile stream
  int obuf;               // O^T buffers in TMEM (2: a split's O is written out one tile late)
  int nbuf;           // K/V ring slots (32 KB each)
  float c2;
  unsigned long long timeout_ns;
  LogitExt ext;       // sinks unused: the merge adds them
  // K/V view: per-sequence lengths and paging (both optional)
  const int* seq_lens;     // [B] or nullptr: every sequence has Skv keys
  const int* block_table;  // [B, max_pages] or nullptr: unpaged
  int max_pages, page_size;
  int mask_rows;           // query rows whose mask values are staged in shared memory (0: none)
  // fp8 e4m3 K/V: one scale per K/V head (K = code * k_scale[kvh], same for V)
  const float* k_scale;
  const float* v_scale;
  // query rows per CTA (Sq for decode; fewer when a long Sq is cut into
  // chunks, one CTA row of the grid each: nqc chunks)
  int qchunk, nqc;
  // final output instead of partials (one split): O [B, Sq, Hq, D] as bf16
  // (fout_bf16) or fp32 at fout, LSE at part_lse (may be nullptr)
  void* fout;
  int fout_bf16;
  // V is a view of K (same base and strides): K tiles stay in L2 (evict_last)
  // until their V reads, which then drop them (evict_first)
  int kv_shared;
  // 1: the num_splits CTAs of one (b, kvh) run as one thread-block cluster
  // and merge their key ranges through distributed shared memory: final O at
  // fout and LSE at part_lse ([B, Hq, Sq]), no partials (group must be 1)
  int cmerge;
};

struct MergeParams {
  const float* part_out;
  const float* part_lse;
  void* out;
  float* lse;
  const float* sinks;  // [Hq] or nullptr
  int B, Hq, Sq, D, num_splits, out_f32;
};

// Each returns a cudaError_t value (as int) from the launch.
// D: the Q and K head size; Dv: the V and O head size (D = Dv in 64, 128,
// 256, or D = 192 with Dv = 128)
int launch_prefill(int D, int Dv, bool ext, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                   const CUtensorMap& tm, const PrefillParams& p, cudaStream_t stream);
size_t prefill_smem_bytes(int D, int Dv);
// The CTA-pair prefill (D = Dv = 256, even Hq/Hkv, no additive mask): each
// cluster of two CTAs runs the two query heads of a K/V group; tk64 tiles K
// in boxes of 64 keys (64 columns x 64 rows), tv and tq as for launch_prefill.
// p.units_per_kvh must be (Hq/Hkv)/2.
int launch_prefill_pair(int D, bool ext, const CUtensorMap& tq, const CUtensorMap& tk64, const CUtensorMap& tv,
                        const PrefillParams& p, cudaStream_t stream);
// D: the Q and K head size; Dv: the V and O head size (pairs with D != Dv:
// 576/512, 320/256, 192/128, bf16 only)
int launch_decode_split(int D, int Dv, bool ext, bool fp8, const CUtensorMap& tq, const CUtensorMap& tk,
                        const CUtensorMap& tv, const DecodeParams& p, cudaStream_t stream);
bool decode_dims_supported(int D, int Dv, bool fp8);
size_t decode_smem_bytes(int D, int RP, int nbuf, int mask_rows, bool fp8);
int decode_max_group();
int decode_max_cluster();
int launch_merge(const MergeParams& p, cudaStream_t stream);
int launch_watchdog_selftest(int* status, unsigned long long limit_ns, cudaStream_t stream);

}  // namespace gqa
