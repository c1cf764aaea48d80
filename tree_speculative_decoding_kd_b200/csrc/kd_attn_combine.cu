// Split-KV merge: each key-range partition s of a row produced a normalised
// partial output o_s and its log-sum-exp lse_s.  The row's result is
//   LSE = ln sum_s exp(lse_s),   out = sum_s exp(lse_s - LSE) * o_s,
// the log-sum-exp identity for a softmax taken over a union of disjoint key sets.
// One warp per (request, node, head) row; each lane owns 16 latent columns.

#include <math.h>

#include "kd_common.cuh"
#include "kd_ptx.cuh"

namespace kd {

__global__ void __launch_bounds__(128)
combine_kernel(const float* __restrict__ part_o, const float* __restrict__ part_lse,
               const int32_t* __restrict__ cache_lens, int64_t rows, int n, int H, int64_t cap,
               int splits, uint16_t* __restrict__ out, float* __restrict__ lse) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int64_t b = row / ((int64_t)n * H);
  const int64_t L = cache_lens[b];
  if (L < 0 || L + n > cap) return;        // request skipped by the attention kernel
  const float LOG2E = 1.4426950408889634f;
  float mx = -INFINITY;
  for (int s = 0; s < splits; ++s) mx = fmaxf(mx, part_lse[(int64_t)s * rows + row]);
  float acc[16];
#pragma unroll
  for (int k = 0; k < 16; ++k) acc[k] = 0.f;
  float sum = 0.f;
  if (mx != -INFINITY) {
    // four partitions at a time: all of their loads are issued before any is used,
    // so a row's partials stream in together rather than one round trip per partition
    for (int s0 = 0; s0 < splits; s0 += 4) {
      float4 v[4][4];
      float wgt[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int s = s0 + j < splits ? s0 + j : s0;        // past the end: reload s0 at weight 0
        const float4* src = reinterpret_cast<const float4*>(part_o + ((int64_t)s * rows + row) * KD_D_C + lane * 16);
#pragma unroll
        for (int q = 0; q < 4; ++q) v[j][q] = src[q];
        const float ls = part_lse[(int64_t)s * rows + row];
        wgt[j] = s0 + j < splits ? ptx::ex2((ls - mx) * LOG2E) : 0.f;   // 0 for an empty partition
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        sum += wgt[j];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          acc[4 * q + 0] = fmaf(wgt[j], v[j][q].x, acc[4 * q + 0]);
          acc[4 * q + 1] = fmaf(wgt[j], v[j][q].y, acc[4 * q + 1]);
          acc[4 * q + 2] = fmaf(wgt[j], v[j][q].z, acc[4 * q + 2]);
          acc[4 * q + 3] = fmaf(wgt[j], v[j][q].w, acc[4 * q + 3]);
        }
      }
    }
  }
  const float inv = sum > 0.f ? 1.f / sum : 0.f;
  uint32_t pk[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) pk[k] = ptx::pack_bf16x2(acc[2 * k] * inv, acc[2 * k + 1] * inv);
  uint4* op = reinterpret_cast<uint4*>(out + row * KD_D_C + lane * 16);
  op[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
  op[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
  if (lane == 0) lse[row] = sum > 0.f ? mx + __logf(sum) : -INFINITY;
}

int launch_combine(const float* part_o, const float* part_lse, const int32_t* cache_lens, int B,
                   int n, int H, int64_t cap, int splits, uint16_t* out, float* lse,
                   cudaStream_t stream) {
  const int64_t rows = (int64_t)B * n * H;
  const int64_t blocks = (rows + 3) / 4;
  combine_kernel<<<(unsigned)blocks, 128, 0, stream>>>(part_o, part_lse, cache_lens, rows, n, H,
                                                        cap, splits, out, lse);
  return launch_status("combine_kernel");
}

}  // namespace kd
