// Merge of split-KV partials by their log-sum-exp, plus the watchdog self-test.
//
// For each output row: M = max_s lse_s, w_s = exp(lse_s - M),
// out = sum_s w_s O_s / sum_s w_s, lse = M + log(sum_s w_s); splits that
// published lse = -inf carry weight 0; an optional sink logit joins M and the
// denominator only ("Anbeeld/beellama.cpp PR #149", review
// of the combine kernel that merges per-block partials for parallel_blocks > 1).
//
// Memory-bound: a block owns 128 consecutive columns of one row, each lane a
// float4 of them, so a warp reads 512 contiguous bytes of a split's partial
// row; the block's four warps take every fourth split.
#include "kernels.h"
#include "ptx.cuh"

namespace gqa {
namespace {

__global__ void __launch_bounds__(128, 8) merge_kernel(const MergeParams p) {
  // One block per (row, 128-column chunk).  Warp w accumulates splits
  // w, w+4, w+8, ... (lane = one float4 of the chunk), so all of a row-chunk's
  // partial loads are in flight at once; the four warps' sums are combined in
  // shared memory.
  __shared__ float4 part_acc[3][32];
  __shared__ float part_w[3], part_m[3];
  // launched as a dependent of the split kernel: its partials are complete
  // and visible past this point
  griddep_wait();
  const int f4_per_row = p.D / 4;
  const int chunks = (f4_per_row + 31) / 32;
  const long long blk = blockIdx.x;
  const long long row = blk / chunks;                // (b, s, h) in O order
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int f = (int)(blk - row * chunks) * 32 + lane;
  const bool active = f < f4_per_row;
  const int h = (int)(row % p.Hq);
  const int s = (int)((row / p.Hq) % p.Sq);
  const int b = (int)(row / ((long long)p.Hq * p.Sq));
  const size_t lse_row = ((size_t)b * p.Hq + h) * p.Sq + s;
  const size_t lse_stride = (size_t)p.B * p.Hq * p.Sq;
  const size_t out_stride4 = (size_t)p.B * p.Sq * p.Hq * p.D / 4;
  const float4* src = reinterpret_cast<const float4*>(p.part_out + (size_t)row * p.D) + (active ? f : 0);

  // Warp w merges splits w, w+4, ... against its own running maximum Mw of
  // their LSEs (eight loads in flight per batch, issued before any
  // arithmetic); the four warps' (Mw, sum, acc) then combine against the
  // common M, which the sink logit joins (the sink adds only to the
  // denominator).  Every lane of a warp loads the same LSEs, so Mw is
  // warp-uniform.
  constexpr float L2E = 1.4426950408889634f;
  const float sink = p.sinks != nullptr ? __ldg(p.sinks + h) : -INFINITY;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float wsum = 0.f, Mw = -INFINITY;
  for (int s0 = warp; s0 < p.num_splits; s0 += 32) {
    float4 o[8];
    float x[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int sg = s0 + 4 * u;
      if (sg < p.num_splits) {
        o[u] = __ldg(src + (size_t)sg * out_stride4);
        x[u] = __ldg(p.part_lse + sg * lse_stride + lse_row);
      } else {
        o[u] = make_float4(0.f, 0.f, 0.f, 0.f);
        x[u] = -INFINITY;
      }
    }
    float mb = Mw;
#pragma unroll
    for (int u = 0; u < 8; ++u) mb = fmaxf(mb, x[u]);
    if (mb != Mw) {   // the batch raised the maximum: rescale what came before
      const float a = (Mw == -INFINITY) ? 0.f : ex2_approx((Mw - mb) * L2E);
      wsum *= a;
      acc.x *= a;
      acc.y *= a;
      acc.z *= a;
      acc.w *= a;
      Mw = mb;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if (x[u] != -INFINITY) {
        const float w = ex2_approx((x[u] - Mw) * L2E);
        wsum += w;
        acc.x = fmaf(w, o[u].x, acc.x);
        acc.y = fmaf(w, o[u].y, acc.y);
        acc.z = fmaf(w, o[u].z, acc.z);
        acc.w = fmaf(w, o[u].w, acc.w);
      }
    }
  }
  if (warp > 0) {
    part_acc[warp - 1][lane] = acc;
    if (lane == 0) {
      part_w[warp - 1] = wsum;
      part_m[warp - 1] = Mw;
    }
  }
  __syncthreads();
  if (warp != 0) return;
  float M = fmaxf(Mw, sink);
#pragma unroll
  for (int i = 0; i < 3; ++i) M = fmaxf(M, part_m[i]);
  {
    const float a = (Mw == -INFINITY) ? 0.f : ex2_approx((Mw - M) * L2E);
    wsum *= a;
    acc.x *= a;
    acc.y *= a;
    acc.z *= a;
    acc.w *= a;
  }
#pragma unroll
  for (int i = 0; i < 3; ++i) {
    const float mi = part_m[i];
    const float a = (mi == -INFINITY) ? 0.f : ex2_approx((mi - M) * L2E);
    const float4 q = part_acc[i][lane];
    acc.x = fmaf(a, q.x, acc.x);
    acc.y = fmaf(a, q.y, acc.y);
    acc.z = fmaf(a, q.z, acc.z);
    acc.w = fmaf(a, q.w, acc.w);
    wsum = fmaf(a, part_w[i], wsum);
  }
  if (sink != -INFINITY) wsum += ex2_approx((sink - M) * L2E);
  if (M != -INFINITY) {
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
  const long long blocks = (long long)p.B * p.Sq * p.Hq * chunks;
  if (blocks <= 0 || blocks > 0x7fffffffLL) return (int)cudaErrorInvalidValue;
  // Programmatic stream serialization: the merge grid may be scheduled while
  // the kernel before it on the stream (the split kernel, which allows it
  // from the start of each CTA) is still running; every block waits at
  // griddep_wait() until that kernel has completed.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)blocks);
  cfg.blockDim = dim3(128);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, merge_kernel, p);
  if (e != cudaSuccess) return (int)e;
  return (int)cudaGetLastError();
}

int launch_watchdog_selftest(int* status, unsigned long long limit_ns, cudaStream_t stream) {
  watchdog_selftest_kernel<<<1, 32, 0, stream>>>(status, limit_ns);
  return (int)cudaGetLastError();
}

}  // namespace gqa
