// merge_kernel.cuh — merge attention results computed over disjoint key sets.
//
// Each part r holds, for every query row, the normalised output O_r and the
// log-sum-exp LSE_r of the scores against its own keys. The combined result
// rescales every part to the common maximum before adding ("Chapter 3: MHA
// Limitations, MQA, GQA, and FlashAttention", section 3.5):
//   M = max_r LSE_r,  w_r = exp(LSE_r - M),  L = sum_r w_r,
//   O = sum_r w_r O_r / L,  LSE = M + ln L,
// and a row no part saw a key for gets O = 0, LSE = -inf. Used to assemble
// sequence-sharded (context-parallel) attention from per-shard results.
#pragma once

#include <cuda_bf16.h>
#include <math_constants.h>

#include "sm100_ptx.cuh"

namespace attn {

// One warp per (b, query row, head): lane l owns elements [4l, 4l + 4) (D = 128)
// or [2l, 2l + 2) (D = 64). Parts: o_parts [R][B, Nq, H, D] f32, lse_parts
// [R][B, H, Nq] f32; outputs o [B, Nq, H, D] bf16, lse [B, H, Nq] (or null).
// All parts' LSEs, then all parts' rows, are loaded as independent requests
// (RMAX >= R parts; a part with LSE = -inf gets weight exp(-inf) = 0).
template <int D, int RMAX>
__global__ void __launch_bounds__(256) attn_merge_kernel(const float* __restrict__ o_parts,
                                                         const float* __restrict__ lse_parts,
                                                         int R, uint16_t* __restrict__ o,
                                                         float* __restrict__ lse, int B, int Nq,
                                                         int H) {
  constexpr int EPL = D / 32;
  const long long row = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const long long rows = static_cast<long long>(B) * Nq * H;
  if (row >= rows) return;
  const int h = int(row % H);
  const long long bq = row / H;                               // b * Nq + q
  const int q = int(bq % Nq), b = int(bq / Nq);
  const size_t lrow = (size_t(b) * H + h) * Nq + q;           // index in [B, H, Nq]
  const size_t part_o = size_t(rows) * D, part_l = size_t(rows);
  float lr[RMAX];
#pragma unroll
  for (int r = 0; r < RMAX; ++r) lr[r] = r < R ? __ldg(lse_parts + r * part_l + lrow) : -CUDART_INF_F;
  float M = -CUDART_INF_F;
#pragma unroll
  for (int r = 0; r < RMAX; ++r) M = fmaxf(M, lr[r]);
  float acc[EPL];
#pragma unroll
  for (int e = 0; e < EPL; ++e) acc[e] = 0.f;
  float L = 0.f;
  if (M > -CUDART_INF_F) {
    float v[RMAX][EPL];
#pragma unroll
    for (int r = 0; r < RMAX; ++r) {
      if (r < R) {
        const float* src = o_parts + r * part_o + size_t(row) * D + lane * EPL;
        if constexpr (EPL == 4) {
          const float4 x = __ldg(reinterpret_cast<const float4*>(src));
          v[r][0] = x.x; v[r][1] = x.y; v[r][2] = x.z; v[r][3] = x.w;
        } else {
          const float2 x = __ldg(reinterpret_cast<const float2*>(src));
          v[r][0] = x.x; v[r][1] = x.y;
        }
      }
    }
#pragma unroll
    for (int r = 0; r < RMAX; ++r) {
      if (r < R) {
        const float w = expf(lr[r] - M);                      // 0 for a part with no key
        L += w;
#pragma unroll
        for (int e = 0; e < EPL; ++e) acc[e] = fmaf(w, v[r][e], acc[e]);
      }
    }
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  uint16_t* dst = o + size_t(row) * D + lane * EPL;
  if constexpr (EPL == 4) {
    *reinterpret_cast<uint2*>(dst) = make_uint2(pack_bf16x2(acc[0] * inv, acc[1] * inv),
                                                pack_bf16x2(acc[2] * inv, acc[3] * inv));
  } else {
    *reinterpret_cast<uint32_t*>(dst) = pack_bf16x2(acc[0] * inv, acc[1] * inv);
  }
  if (lane == 0 && lse != nullptr) lse[lrow] = L > 0.f ? M + logf(L) : -CUDART_INF_F;
}

}  // namespace attn
