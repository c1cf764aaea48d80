// Target argmax over each tree node's logits, fused with greedy acceptance.
//
// Sources (page title, section):
//   "The Architecture of Pragmatic Ambition" -- "The Output Knowledge: What This
//       Message Creates": argmax is one of the engine's primitives, and the
//       speculative output must equal greedy decoding token for token, so the
//       target's token after a node is the argmax of its logits there;
//       "The Knowledge Architecture": the greedy walk to the longest prefix that
//       matches those tokens.
//
// Reading logits [B][n][V] once is the whole cost (HBM bound: 4·V bytes per node).
// One CTA streams one 64 KB chunk of one node's row with coalesced 16-byte loads,
// sixteen in flight per thread.  Each thread keeps its 64 values in registers and
// takes their NaN-propagating max (a third of an instruction per value); the CTA then
// agrees on the chunk's maximum, and only the threads that hold it scan their values
// from the highest index down for it (or for a NaN), so that the last hit is the
// lowest index; -0.0 == +0.0 there.  Ranks compare as 64-bit words: the value's
// order-preserving key in the high word, the complement of the index in the low word,
// so that one unsigned max picks the largest value and, among equal values, the
// lowest index.  NaN ranks above every number and -0.0 ranks as +0.0.  The chunk's rank is merged into the row's by atomicMax; the
// last CTA of a request (counted per request) turns the n ranks into tokens and
// runs the greedy walk with one warp.

#include "kd_common.cuh"
#include "kd_accept.cuh"

namespace kd {

constexpr int AM_THREADS = 256;
constexpr int AM_VEC = 16;                                 // 16-byte loads per thread per chunk
constexpr int AM_CHUNK = AM_THREADS * AM_VEC * 4;          // 16384 logits = 64 KB per CTA

// Order-preserving key of a logit (see above).
__device__ __forceinline__ uint32_t logit_key(float x) {
  uint32_t u = __float_as_uint(x);
  if ((u & 0x7fffffffu) > 0x7f800000u) return 0xffffffffu;   // NaN: above every number
  if (u == 0x80000000u) u = 0u;                              // -0.0 ranks as +0.0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);         // monotone in the value
}

__device__ __forceinline__ float max_nan3(float a, float b, float c) {
  float d;
  asm("max.NaN.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

__device__ __forceinline__ unsigned long long umax64(unsigned long long a, unsigned long long b) {
  return a > b ? a : b;
}

__global__ void __launch_bounds__(AM_THREADS, 3)
argmax_accept_kernel(const float* __restrict__ logits, int64_t V, int chunks, int n,
                     const int32_t* __restrict__ tokens, const int32_t* __restrict__ parents,
                     int32_t* argmax, unsigned long long* best, unsigned int* done,
                     int32_t* __restrict__ path, int32_t* __restrict__ len,
                     int32_t* __restrict__ bonus, int32_t* dev_error) {
  const int64_t row = blockIdx.x / chunks;
  const int chunk = blockIdx.x % chunks;
  const int b = (int)(row / n);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float4* src = reinterpret_cast<const float4*>(logits + row * V);
  const int64_t e0 = (int64_t)chunk * AM_CHUNK + (int64_t)threadIdx.x * 4;

  // all sixteen loads first (V is a multiple of 4, so a vector is either wholly inside
  // the row or wholly past its end; past the end reads as -inf and is never chosen)
  const float NEG = -INFINITY;
  float4 x[AM_VEC];
#pragma unroll
  for (int j = 0; j < AM_VEC; ++j) {
    const int64_t e = e0 + (int64_t)j * AM_THREADS * 4;
    x[j] = e < V ? __ldcs(src + (e >> 2)) : make_float4(NEG, NEG, NEG, NEG);
  }
  float mv = x[0].x;
#pragma unroll
  for (int j = 0; j < AM_VEC; ++j) mv = max_nan3(max_nan3(mv, x[j].x, x[j].y), x[j].z, x[j].w);
  // the chunk's maximum key (a thread whose elements all lie past V holds -inf, which
  // only wins if every real element is -inf too, and then the scan below skips it)
  uint32_t k = logit_key(mv);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) k = max(k, __shfl_xor_sync(0xffffffffu, k, off));
  __shared__ uint32_t wk[AM_THREADS / 32];
  __shared__ unsigned long long wm[AM_THREADS / 32];
  __shared__ int last;
  if (lane == 0) wk[warp] = k;
  __syncthreads();
  uint32_t kmax = wk[0];
#pragma unroll
  for (int w = 1; w < AM_THREADS / 32; ++w) kmax = max(kmax, wk[w]);
  // only threads holding it look for its lowest index: scan down, the last hit wins
  unsigned long long m = 0ull;                             // below every real rank
  if (logit_key(mv) == kmax) {
    const bool want_nan = mv != mv;
    const bool whole = e0 + (int64_t)(AM_VEC - 1) * AM_THREADS * 4 < V;   // no element past V
    uint32_t idx = 0xffffffffu;
#pragma unroll
    for (int j = AM_VEC - 1; j >= 0; --j) {
      const int64_t e = e0 + (int64_t)j * AM_THREADS * 4;
      const bool in = whole || e < V;
      const uint32_t i = (uint32_t)e;
      const float v[4] = {x[j].x, x[j].y, x[j].z, x[j].w};
#pragma unroll
      for (int c = 3; c >= 0; --c) {
        const bool hit = want_nan ? (v[c] != v[c]) : (v[c] == mv);
        idx = (hit && in) ? i + c : idx;
      }
    }
    if (idx != 0xffffffffu) m = ((unsigned long long)kmax << 32) | (unsigned long long)(0xffffffffu - idx);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = umax64(m, __shfl_xor_sync(0xffffffffu, m, off));
  if (lane == 0) wm[warp] = m;
  __syncthreads();
  if (warp != 0) return;
  m = lane < AM_THREADS / 32 ? wm[lane] : 0ull;
#pragma unroll
  for (int off = 4; off > 0; off >>= 1) m = umax64(m, __shfl_xor_sync(0xffffffffu, m, off));
  if (lane == 0) {
    atomicMax(best + row, m);
    __threadfence();                                       // the rank is visible before the count
    last = atomicAdd(done + b, 1u) == (unsigned)(n * chunks - 1);
  }
  __syncwarp();
  if (!last) return;
  // last CTA of request b: every other CTA's rank has landed (they fenced before counting)
  __threadfence();
  for (int i = lane; i < n; i += 32) {
    const unsigned long long r = __ldcg(best + (size_t)b * n + i);
    argmax[(size_t)b * n + i] = (int32_t)(0xffffffffu - (uint32_t)r);
  }
  __syncwarp();
  __threadfence_block();
  accept_walk(tokens, parents, argmax, b, n, path, len, bonus, dev_error);
}

// Workspace: per-node ranks (8 B), per-request counters (4 B), and the tokens when
// the caller does not want them back (4 B per node).
static size_t ws_layout(int B, int n, size_t* off_done, size_t* off_tok) {
  const size_t rows = (size_t)B * n;
  *off_done = rows * 8;
  *off_tok = ((*off_done + (size_t)B * 4 + 15) / 16) * 16;
  return *off_tok + rows * 4;
}

}  // namespace kd

using namespace kd;

extern "C" size_t kd_accept_workspace_bytes(int B, int n) {
  if (!shapes_ok(B, n)) return 0;
  size_t od, ot;
  return ws_layout(B, n, &od, &ot);
}

extern "C" int kd_tree_accept_logits(const int32_t* node_tokens, const int32_t* parents,
                                     const float* logits, int B, int n, int64_t V,
                                     int32_t* target_argmax, int32_t* path, int32_t* len,
                                     int32_t* bonus, void* workspace, size_t ws_bytes,
                                     int32_t* dev_error, cudaStream_t stream) {
  if (!node_tokens || !parents || !logits || !path || !len || !bonus || !workspace ||
      !shapes_ok(B, n) || V < 4 || (V & 3) || V > (int64_t)INT32_MAX || !aligned16(logits) ||
      (reinterpret_cast<uintptr_t>(workspace) & 15u))
    return KD_EINVAL;
  size_t off_done, off_tok;
  const size_t need = ws_layout(B, n, &off_done, &off_tok);
  if (ws_bytes < need) return KD_ERANGE;
  const int64_t chunks = (V + AM_CHUNK - 1) / AM_CHUNK;
  const int64_t grid = (int64_t)B * n * chunks;
  if (grid > INT32_MAX) return KD_EINVAL;
  int st = device_sms(nullptr);
  if (st) return st;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  st = cuda_status(cudaMemsetAsync(ws, 0, off_tok, stream), "cudaMemsetAsync(accept workspace)");
  if (st) return st;
  int32_t* am = target_argmax ? target_argmax : reinterpret_cast<int32_t*>(ws + off_tok);
  argmax_accept_kernel<<<(unsigned)grid, AM_THREADS, 0, stream>>>(
      logits, V, (int)chunks, n, node_tokens, parents, am,
      reinterpret_cast<unsigned long long*>(ws), reinterpret_cast<unsigned int*>(ws + off_done), path,
      len, bonus, dev_error);
  return launch_status("argmax_accept_kernel");
}
