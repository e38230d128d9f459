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
  __shared__ float part_w[3];
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

  // max of the split LSEs and the sink logit (every warp computes it; the
  // loads are tiny); the sink joins only the denominator
  const float sink = p.sinks != nullptr ? __ldg(p.sinks + h) : -INFINITY;
  float M = sink;
  for (int sg = lane; sg < p.num_splits; sg += 32) M = fmaxf(M, __ldg(p.part_lse + sg * lse_stride + lse_row));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));

  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float wsum = 0.f;
  // this warp's splits, eight loads in flight per batch; the loads do not
  // wait for the maximum above (every published partial is finite)
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
        x[u] = -INFINITY;
      }
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if (x[u] != -INFINITY) {
        const float w = ex2_approx((x[u] - M) * 1.4426950408889634f);
        wsum += w;
        acc.x = fmaf(w, o[u].x, acc.x);
        acc.y = fmaf(w, o[u].y, acc.y);
        acc.z = fmaf(w, o[u].z, acc.z);
        acc.w = fmaf(w, o[u].w, acc.w);
      }
    }
  }
  if (warp == 0 && sink != -INFINITY) wsum += ex2_approx((sink - M) * 1.4426950408889634f);
  if (warp > 0) {
    part_acc[warp - 1][lane] = acc;
    if (lane == 0) part_w[warp - 1] = wsum;
  }
  __syncthreads();
  if (warp != 0) return;
#pragma unroll
  for (int i = 0; i < 3; ++i) {
    const float4 a = part_acc[i][lane];
    acc.x += a.x;
    acc.y += a.y;
    acc.z += a.z;
    acc.w += a.w;
    wsum += part_w[i];
  }
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
  merge_kernel<<<(unsigned)blocks, 128, 0, stream>>>(p);
  return (int)cudaGetLastError();
}

int launch_watchdog_selftest(int* status, unsigned long long limit_ns, cudaStream_t stream) {
  watchdog_selftest_kernel<<<1, 32, 0, stream>>>(status, limit_ns);
  return (int)cudaGetLastError();
}

}  // namespace gqa
