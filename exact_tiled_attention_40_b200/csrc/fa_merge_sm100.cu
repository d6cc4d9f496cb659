// Merge of two partial attention results over disjoint key sets, by their LSE.
//
// unite.ai, "Flash Attention: Revolutionizing Transformer Efficiency", section
// "The Mathematics of Flash Attention": the softmax over a concatenation of key
// blocks follows from each block's maximum and sum.  With normalised partial
// outputs O_a, O_b and their log-sum-exps lse_a, lse_b:
//     lse = log(e^lse_a + e^lse_b),  O = e^(lse_a - lse) O_a + e^(lse_b - lse) O_b.
// The sequence-sharded forward folds each key chunk's result into an fp32
// accumulator with this kernel.  HBM-bound: a warp per row, D / 32 values per
// lane, every load and store coalesced.
#include <algorithm>
#include <cmath>
#include <cstdint>

#include "fa_internal.h"
#include "../../include/fa.h"

namespace fa {
namespace {

constexpr int kMergeThreads = 256;

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
__device__ __forceinline__ uint32_t to_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

template <int D>
__global__ void __launch_bounds__(kMergeThreads)
    fa_merge_kernel(float* __restrict__ o_acc, float* __restrict__ lse_acc,
                    const uint16_t* __restrict__ o_part, const float* __restrict__ lse_part,
                    uint16_t* __restrict__ o_out, long long rows, int first) {
  constexpr int E = D / 32;
  const int lane = threadIdx.x & 31;
  const long long warps = static_cast<long long>(gridDim.x) * (kMergeThreads / 32);
  for (long long row = static_cast<long long>(blockIdx.x) * (kMergeThreads / 32) +
                       (threadIdx.x >> 5);
       row < rows; row += warps) {
    const size_t base = static_cast<size_t>(row) * D + lane * E;
    float ob[E];
    if constexpr (E == 4) {
      const uint2 u = __ldg(reinterpret_cast<const uint2*>(o_part + base));
      ob[0] = bf16_lo(u.x);
      ob[1] = bf16_hi(u.x);
      ob[2] = bf16_lo(u.y);
      ob[3] = bf16_hi(u.y);
    } else {
      const uint32_t u = __ldg(reinterpret_cast<const uint32_t*>(o_part + base));
      ob[0] = bf16_lo(u);
      ob[1] = bf16_hi(u);
    }
    const float lb = __ldg(lse_part + row);
    float o[E];
    float l;
    if (first) {
#pragma unroll
      for (int e = 0; e < E; ++e) o[e] = ob[e];
      l = lb;
    } else {
      float oa[E];
      if constexpr (E == 4) {
        const float4 a = *reinterpret_cast<const float4*>(o_acc + base);
        oa[0] = a.x;
        oa[1] = a.y;
        oa[2] = a.z;
        oa[3] = a.w;
      } else {
        const float2 a = *reinterpret_cast<const float2*>(o_acc + base);
        oa[0] = a.x;
        oa[1] = a.y;
      }
      const float la = lse_acc[row];
      const float m = fmaxf(la, lb);
      if (m == -INFINITY) {          // neither part saw a key: O stays 0
#pragma unroll
        for (int e = 0; e < E; ++e) o[e] = 0.f;
        l = -INFINITY;
      } else {
        float wa = expf(la - m), wb = expf(lb - m);
        const float s = wa + wb;
        l = m + logf(s);
        wa /= s;
        wb /= s;
#pragma unroll
        for (int e = 0; e < E; ++e) o[e] = wa * oa[e] + wb * ob[e];
      }
    }
    if constexpr (E == 4)
      *reinterpret_cast<float4*>(o_acc + base) = make_float4(o[0], o[1], o[2], o[3]);
    else
      *reinterpret_cast<float2*>(o_acc + base) = make_float2(o[0], o[1]);
    if (lane == 0) lse_acc[row] = l;
    if (o_out) {
      if constexpr (E == 4)
        *reinterpret_cast<uint2*>(o_out + base) =
            make_uint2(to_bf16x2(o[0], o[1]), to_bf16x2(o[2], o[3]));
      else
        *reinterpret_cast<uint32_t*>(o_out + base) = to_bf16x2(o[0], o[1]);
    }
  }
}

}  // namespace

int launch_merge_partials(float* o_acc, float* lse_acc, const void* o_part, const float* lse_part,
                          void* o_out, long long rows, int D, int first, cudaStream_t stream,
                          int device) {
  const int nsm = device_sm_count(device);
  if (nsm <= 0) return set_error(FA_ERR_CUDA, "cannot read the SM count of device %d", device);
  const long long per_block = kMergeThreads / 32;
  const long long want = (rows + per_block - 1) / per_block;
  const int grid = static_cast<int>(std::min<long long>(want, 8LL * nsm));
  if (grid == 0) return FA_OK;
  const auto* op = static_cast<const uint16_t*>(o_part);
  auto* oo = static_cast<uint16_t*>(o_out);
  if (D == 128)
    fa_merge_kernel<128><<<grid, kMergeThreads, 0, stream>>>(o_acc, lse_acc, op, lse_part, oo,
                                                             rows, first);
  else
    fa_merge_kernel<64><<<grid, kMergeThreads, 0, stream>>>(o_acc, lse_acc, op, lse_part, oo,
                                                            rows, first);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess)
    return set_error(FA_ERR_CUDA, "fa_merge_partials launch: %s", cudaGetErrorString(e));
  return FA_OK;
}

}  // namespace fa
