// CUDA-core tree-verify attention: one warp per (request, node, head), keys
// streamed one row at a time with an online softmax.  It uses no tensor cores and
// exists as a plain second GPU implementation for bring-up and cross-checks; the
// tensor-core kernel in kd_attn_tc.cu is the product path.
//
// Definition ("The Architecture of Pragmatic Ambition", sections "The Thinking
// Process" -- absorb form -- and "The Knowledge Architecture" -- visibility-masked
// tree attention): node i of request b sees slots 0..L-1 and slots L+k for every
// k set in its mask; score = scale * (q_abs . c_kv + q_rope . k_rope); value = c_kv.

#include <math.h>

#include "kd_common.cuh"
#include "kd_ptx.cuh"

namespace kd {

__device__ __forceinline__ float bf_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// Checks shared by both attention kernels for one row: root and own bit in the
// mask, position = L + depth when positions are given.
__device__ __forceinline__ void check_node_row(const uint32_t* w, int W, int i, int64_t L,
                                               const int32_t* positions, int64_t pos_idx,
                                               int32_t* err) {
  int depth = -1;
  for (int q = 0; q < W; ++q) depth += __popc(w[q]);
  const bool bad_mask = !(w[0] & 1u) || !((w[i >> 5] >> (i & 31)) & 1u);
  if (bad_mask) raise_dev_error(err, KD_DEV_BAD_MASK);
  if (positions && positions[pos_idx] != (int32_t)(L + depth))
    raise_dev_error(err, KD_DEV_BAD_POSITION);
}

__global__ void __launch_bounds__(256)
attn_simt_kernel(const uint16_t* __restrict__ q_abs, const uint16_t* __restrict__ q_rope,
                 const uint16_t* __restrict__ c_kv, const uint16_t* __restrict__ k_rope,
                 int64_t sc, int64_t sr, int64_t cap, const int32_t* __restrict__ cache_lens,
                 const uint32_t* __restrict__ vis, const int32_t* __restrict__ positions, int n,
                 int H, float scale_log2, uint16_t* __restrict__ out, float* __restrict__ lse,
                 int32_t* err) {
  const int lane = threadIdx.x & 31;
  const int h = blockIdx.y * 8 + (threadIdx.x >> 5);
  const int bi = blockIdx.x;           // b * n + i
  const int b = bi / n, i = bi % n;
  if (h >= H) return;
  const int64_t L = cache_lens[b];
  if (L < 0 || L + n > cap) {
    if (lane == 0 && h == 0) raise_dev_error(err, KD_DEV_CACHE_FULL);
    return;
  }
  const int W = (n + 31) >> 5;
  uint32_t w[4] = {0, 0, 0, 0};
  for (int q = 0; q < W; ++q) w[q] = vis[(size_t)bi * W + q];
  if (lane == 0 && h == 0) check_node_row(w, W, i, L, positions, bi, err);

  // lane owns latent dims [16*lane, 16*lane+16) and rope dims [2*lane, 2*lane+2)
  const size_t qrow = (size_t)bi * H + h;
  float qa[16], qr[2];
  {
    const uint4* p = reinterpret_cast<const uint4*>(q_abs + qrow * KD_D_C + lane * 16);
    uint4 v0 = p[0], v1 = p[1];
    uint32_t u[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
    for (int k = 0; k < 8; ++k) { qa[2 * k] = bf_lo(u[k]); qa[2 * k + 1] = bf_hi(u[k]); }
    uint32_t r = *reinterpret_cast<const uint32_t*>(q_rope + qrow * KD_D_R + lane * 2);
    qr[0] = bf_lo(r);
    qr[1] = bf_hi(r);
  }
  float o[16];
#pragma unroll
  for (int k = 0; k < 16; ++k) o[k] = 0.f;
  float m = -INFINITY, l = 0.f;
  const int64_t nkeys = L + n;
  const int64_t row0 = (int64_t)b * cap;
  for (int64_t j = 0; j < nkeys; ++j) {
    if (j >= L) {
      const int k = (int)(j - L);
      if (!((w[k >> 5] >> (k & 31)) & 1u)) continue;
    }
    const uint4* cp = reinterpret_cast<const uint4*>(c_kv + (row0 + j) * sc + lane * 16);
    uint4 v0 = cp[0], v1 = cp[1];
    uint32_t u[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
    float c[16];
#pragma unroll
    for (int k = 0; k < 8; ++k) { c[2 * k] = bf_lo(u[k]); c[2 * k + 1] = bf_hi(u[k]); }
    const uint32_t rr = *reinterpret_cast<const uint32_t*>(k_rope + (row0 + j) * sr + lane * 2);
    float d = qr[0] * bf_lo(rr) + qr[1] * bf_hi(rr);
#pragma unroll
    for (int k = 0; k < 16; ++k) d = fmaf(qa[k], c[k], d);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) d += __shfl_xor_sync(0xffffffffu, d, off);
    const float s2 = d * scale_log2;
    const float mn = fmaxf(m, s2);
    const float corr = ptx::ex2(m - mn);      // 0 when m = -inf
    const float p = ptx::ex2(s2 - mn);
    l = l * corr + p;
#pragma unroll
    for (int k = 0; k < 16; ++k) o[k] = fmaf(o[k], corr, p * c[k]);
    m = mn;
  }
  const float inv = l > 0.f ? 1.f / l : 0.f;
  uint32_t pk[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) pk[k] = ptx::pack_bf16x2(o[2 * k] * inv, o[2 * k + 1] * inv);
  uint4* op = reinterpret_cast<uint4*>(out + qrow * KD_D_C + lane * 16);
  op[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
  op[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
  if (lane == 0) lse[qrow] = l > 0.f ? (m + __log2f(l)) * 0.69314718055994531f : -INFINITY;
}

}  // namespace kd

using namespace kd;

extern "C" int kd_tree_verify_attn_simt(const kd_bf16_t* q_abs, const kd_bf16_t* q_rope,
                                        const kd_bf16_t* c_kv, const kd_bf16_t* k_rope,
                                        int64_t sc, int64_t sr, int64_t cap,
                                        const int32_t* cache_lens, const uint32_t* vis,
                                        const int32_t* positions, int B, int n, int H,
                                        float scale, kd_bf16_t* out, float* lse,
                                        int32_t* dev_error, cudaStream_t stream) {
  if (!q_abs || !q_rope || !cache_lens || !vis || !out || !lse || !shapes_ok(B, n) || H < 1 ||
      H > KD_MAX_HEADS || !cache_ok(c_kv, k_rope, sc, sr, cap) || !aligned16(q_abs) ||
      !aligned16(out) || !(scale > 0.f))
    return KD_EINVAL;
  int st = device_sms(nullptr);
  if (st) return st;
  dim3 grid(B * n, (H + 7) / 8);
  attn_simt_kernel<<<grid, 256, 0, stream>>>(q_abs, q_rope, c_kv, k_rope, sc, sr, cap, cache_lens,
                                             vis, positions, n, H, scale * 1.4426950408889634f,
                                             out, lse, dev_error);
  return launch_status("attn_simt_kernel");
}
