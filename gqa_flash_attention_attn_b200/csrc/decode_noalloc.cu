// Split-KV decode + LSE merge for callers that cannot allocate device memory.
//
// attn_decode_split needs a workspace for its per-split partial outputs and
// log-sum-exps, which the caller normally allocates.  Some callers cannot:
// a plugin host that owns the whole device memory pool and hands an operator
// only its inputs and outputs, or a latency-critical decode loop that must
// never call cudaMalloc (which can synchronise the device).  For them,
// attn_decode_noalloc keeps the partials in a fixed, file-scope device array
// instead, and runs the unchanged split and merge kernels on it.
//
// Properties of that array:
//   - it is ATTN_NOALLOC_SCRATCH_BYTES long and lives in every device that
//     loads this library, from module load until process exit;
//   - host code cannot use its name as a device address: its address is
//     looked up with cudaGetSymbolAddress once per device (with that device
//     current) on the first call made on that device, so make that first call
//     before any stream capture;
//   - every call shares it and it keeps the last call's contents; nothing in
//     it needs to start at zero, because the split kernel writes every partial
//     element that the merge kernel of the same call reads;
//   - calls whose kernels overlap on the GPU (two streams, or two host threads)
//     race on it: serialise them.
#include <cstdint>
#include <mutex>

#include "attn.h"
#include "kernels.h"

namespace {

static __device__ __align__(256) unsigned char g_decode_scratch[ATTN_NOALLOC_SCRATCH_BYTES];

std::mutex g_scratch_mu;
void* g_scratch_dev[64] = {nullptr};

// Device address of the scratch array on the current device (set-up on first use).
void* scratch_on_current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (g_scratch_dev[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr) return nullptr;
    g_scratch_dev[dev] = p;
  }
  return g_scratch_dev[dev];
}

}  // namespace

extern "C" int attn_decode_noalloc(const void* q, const void* k, const void* v, void* out, float* lse, int B,
                                   int Hq, int Hkv, int Sq, int Skv, int D, int q_offset, int causal, float scale,
                                   int num_splits, int out_dtype, void* stream) {
  if (out == nullptr) return ATTN_ERR_INVALID_ARG;
  if (out_dtype != ATTN_BF16 && out_dtype != ATTN_F32) return ATTN_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Sq < 1 || D < 1 || num_splits < 1) return ATTN_ERR_INVALID_ARG;
  // partials: out [S,B,Sq,Hq,D] at offset 0, lse [S,B,Hq,Sq] at the next 256-byte boundary
  const unsigned long long n_out = (unsigned long long)num_splits * B * Sq * Hq * D;
  const unsigned long long n_lse = (unsigned long long)num_splits * B * Hq * Sq;
  const unsigned long long lse_off = (n_out * sizeof(float) + 255ull) & ~255ull;
  if (lse_off + n_lse * sizeof(float) > (unsigned long long)ATTN_NOALLOC_SCRATCH_BYTES) return ATTN_ERR_TOO_LARGE;

  unsigned char* base = static_cast<unsigned char*>(scratch_on_current_device());
  if (base == nullptr) return ATTN_ERR_CUDA;
  float* part_out = reinterpret_cast<float*>(base);
  float* part_lse = reinterpret_cast<float*>(base + lse_off);
  int st = attn_decode_split(q, k, v, part_out, part_lse, B, Hq, Hkv, Sq, Skv, D, q_offset, causal, scale,
                             num_splits, stream);
  if (st != ATTN_OK) return st;
  return attn_merge(part_out, part_lse, out, lse, B, Hq, Sq, D, num_splits, out_dtype, stream);
}
