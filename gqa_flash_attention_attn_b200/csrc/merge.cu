// Merge of split-KV partials by their log-sum-exp, plus the watchdog self-test.
//
// For each output row: M = max_s lse_s, w_s = exp(lse_s - M),
// out = sum_s w_s O_s / sum_s w_s, lse = M + log(sum_s w_s); splits that
// published lse = -inf carry weight 0 ("Anbeeld/beellama.cpp PR #149", review
// of the combine kernel that merges per-block partials for parallel_blocks > 1).
//
// HBM-bound: a warp owns 128 consecutive columns of one row and each lane a
// float4 of them, so a warp reads 512 contiguous bytes of every split's
// partial row, eight splits in flight at a time.
#include "kernels.h"
#include "ptx.cuh"

namespace gqa {
namespace {

__global__ void __launch_bounds__(128) merge_kernel(const MergeParams p) {
  // one warp per (row, 128-column chunk); lane owns one float4 of the chunk
  const int f4_per_row = p.D / 4;
  const int chunks = (f4_per_row + 31) / 32;
  const long long rows = (long long)p.B * p.Sq * p.Hq;
  const long long gw = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (gw >= rows * chunks) return;                  // whole warp leaves together
  const long long row = gw / chunks;                // (b, s, h) in O order
  const int f = (int)(gw - row * chunks) * 32 + lane;
  const bool active = f < f4_per_row;
  const int h = (int)(row % p.Hq);
  const int s = (int)((row / p.Hq) % p.Sq);
  const int b = (int)(row / ((long long)p.Hq * p.Sq));
  const size_t lse_row = ((size_t)b * p.Hq + h) * p.Sq + s;
  const size_t lse_stride = (size_t)p.B * p.Hq * p.Sq;
  const size_t out_stride4 = (size_t)rows * p.D / 4;
  const float4* src = reinterpret_cast<const float4*>(p.part_out + (size_t)row * p.D) + (active ? f : 0);

  // lane i holds lse of splits i, i+32, ...: max over all splits
  float M = -INFINITY;
  for (int sg = lane; sg < p.num_splits; sg += 32) M = fmaxf(M, __ldg(p.part_lse + sg * lse_stride + lse_row));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));

  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float wsum = 0.f;
  if (M != -INFINITY) {
    for (int s0 = 0; s0 < p.num_splits; s0 += 32) {
      const int sg_l = s0 + lane;
      const float x = sg_l < p.num_splits ? __ldg(p.part_lse + sg_l * lse_stride + lse_row) : -INFINITY;
      const float w_l = (x == -INFINITY) ? 0.f : expf(x - M);   // weight of split s0 + lane
      const int n = min(32, p.num_splits - s0);
      int i = 0;
      // eight independent 16-byte loads in flight per lane
      for (; i + 8 <= n; i += 8) {
        float4 o[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) o[u] = __ldg(src + (size_t)(s0 + i + u) * out_stride4);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const float w = __shfl_sync(0xffffffffu, w_l, i + u);
          wsum += w;
          acc.x = fmaf(w, o[u].x, acc.x);
          acc.y = fmaf(w, o[u].y, acc.y);
          acc.z = fmaf(w, o[u].z, acc.z);
          acc.w = fmaf(w, o[u].w, acc.w);
        }
      }
      for (; i < n; ++i) {
        const float4 o = __ldg(src + (size_t)(s0 + i) * out_stride4);
        const float w = __shfl_sync(0xffffffffu, w_l, i);
        wsum += w;
        acc.x = fmaf(w, o.x, acc.x);
        acc.y = fmaf(w, o.y, acc.y);
        acc.z = fmaf(w, o.z, acc.z);
        acc.w = fmaf(w, o.w, acc.w);
      }
    }
    const float inv = 1.f / wsum;
    acc.x *= inv;
    acc.y *= inv;
    acc.z *= inv;
    acc.w *= inv;
  }
  if (active) {
    const size_t o_off = (size_t)row * p.D + 4 * (size_t)f;
    if (p.out_f32) {
      *reinterpret_cast<float4*>(reinterpret_cast<float*>(p.out) + o_off) = acc;
    } else {
      *reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(p.out) + o_off) =
          make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
    }
  }
  if (f == 0 && p.lse != nullptr) p.lse[lse_row] = (M == -INFINITY) ? -INFINITY : M + logf(wsum);
}

// One thread waits on an mbarrier that nothing completes; the bounded wait
// gives up after limit_ns and records the timeout status.
__global__ void watchdog_selftest_kernel(int* status, unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t mbar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&mbar), 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const Watchdog wd{&abort_flag, status, limit_ns};
    (void)mbar_wait(smem_u32(&mbar), 0, wd);
  }
}

}  // namespace

int launch_merge(const MergeParams& p, cudaStream_t stream) {
  const long long chunks = (p.D / 4 + 31) / 32;
  const long long warps = (long long)p.B * p.Sq * p.Hq * chunks;
  const long long blocks = (warps + 3) / 4;
  if (blocks <= 0 || blocks > 0x7fffffffLL) return (int)cudaErrorInvalidValue;
  merge_kernel<<<(unsigned)blocks, 128, 0, stream>>>(p);
  return (int)cudaGetLastError();
}

int launch_watchdog_selftest(int* status, unsigned long long limit_ns, cudaStream_t stream) {
  watchdog_selftest_kernel<<<1, 32, 0, stream>>>(status, limit_ns);
  return (int)cudaGetLastError();
}

}  // namespace gqa
