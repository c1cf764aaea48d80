// Best-first draft-tree construction on the GPU, one warp per request.
//
// Source: "The Architecture of Pragmatic Ambition", section "The Knowledge
// Architecture": the tree builder takes per-depth top-k candidates from a drafter and
// builds a best-first tree for the verify step.  The pages give no scoring rule;
// the reading taken (the plainest one the rest supports):
//   * depth d = 1..D has K candidates (token, log-probability), sorted from the most
//     to the least likely, the same for every path (one distribution per position);
//   * a node's score is the float32 sum of the log-probabilities along its path;
//   * the tree is the root (node 0: the last verified token, depth 0, score 0) plus
//     the n - 1 best nodes, popped one at a time from the frontier of the tree built
//     so far; equal scores go to the lower depth, then the lower parent index, then
//     the lower candidate index; node index = pop order (topological).
// A popped node offers the frontier only its next sibling and its first child: with
// sorted candidates and log-probabilities <= 0 nothing else can score better.
//
// The frontier (at most n entries) lives in shared memory as 64-bit keys whose
// unsigned order is the priority order: the score's order-preserving key, then
// 255 - depth, 255 - parent, 255 - candidate, and the slot in the low byte (the
// triple is unique, so the slot never decides).  A pop is a strided scan plus a
// warp max; lane 0 then writes the node and pushes at most two entries.

#include "kd_common.cuh"

namespace kd {

constexpr int TB_WARPS = 4;                  // requests per CTA
constexpr int TB_FRONT = KD_MAX_NODES + 2;   // each pop removes one entry and adds at most two

__device__ __forceinline__ uint32_t score_key(float x) {
  uint32_t u = __float_as_uint(x);
  if (u == 0x80000000u) u = 0u;                          // -0.0 ranks as +0.0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);     // monotone in the value
}

__device__ __forceinline__ unsigned long long entry_key(float s, int d, int p, int j, int slot) {
  return ((unsigned long long)score_key(s) << 32) | ((uint32_t)(255 - d) << 24) |
         ((uint32_t)(255 - p) << 16) | ((uint32_t)(255 - j) << 8) | (uint32_t)slot;
}

__device__ __forceinline__ unsigned long long umax64(unsigned long long a, unsigned long long b) {
  return a > b ? a : b;
}

__global__ void __launch_bounds__(32 * TB_WARPS)
tree_build_kernel(const float* __restrict__ logp, const int32_t* __restrict__ cand,
                  const int32_t* __restrict__ root, int B, int D, int K, int n,
                  int32_t* __restrict__ parents, int32_t* __restrict__ tokens,
                  int32_t* __restrict__ depth_out, float* __restrict__ score_out) {
  __shared__ unsigned long long fkey[TB_WARPS][TB_FRONT];
  __shared__ float fscore[TB_WARPS][TB_FRONT];
  __shared__ float nscore[TB_WARPS][KD_MAX_NODES];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.x * TB_WARPS + w;
  if (b >= B) return;
  const float* lp = logp + (size_t)b * D * K;
  const int32_t* ct = cand + (size_t)b * D * K;
  unsigned long long* fk = fkey[w];
  float* fs = fscore[w];
  float* ns = nscore[w];
  const size_t o = (size_t)b * n;
  int cnt = (D >= 1 && n > 1) ? 1 : 0;                   // frontier entries (warp-uniform)
  if (lane == 0) {
    parents[o] = -1;
    tokens[o] = root[b];
    if (depth_out) depth_out[o] = 0;
    if (score_out) score_out[o] = 0.f;
    ns[0] = 0.f;
    if (cnt) {
      const float s = lp[0];
      fk[0] = entry_key(s, 1, 0, 0, 0);
      fs[0] = s;
    }
  }
  __syncwarp();
  for (int me = 1; me < n && cnt > 0; ++me) {
    unsigned long long best = 0ull;
    for (int i = lane; i < cnt; i += 32) best = umax64(best, fk[i]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) best = umax64(best, __shfl_xor_sync(0xffffffffu, best, off));
    const int slot = (int)(best & 0xffu);
    const int d = 255 - (int)((best >> 24) & 0xffu);
    const int p = 255 - (int)((best >> 16) & 0xffu);
    const int j = 255 - (int)((best >> 8) & 0xffu);
    const bool sib = j + 1 < K, kid = d < D;
    if (lane == 0) {
      const float s = fs[slot];
      const int last = cnt - 1;
      if (slot != last) {                               // the last entry fills the hole
        fk[slot] = (fk[last] & ~0xffull) | (unsigned long long)slot;
        fs[slot] = fs[last];
      }
      parents[o + me] = p;
      tokens[o + me] = ct[(size_t)(d - 1) * K + j];
      if (depth_out) depth_out[o + me] = d;
      if (score_out) score_out[o + me] = s;
      ns[me] = s;
      int c = last;
      if (sib) {                                        // next sibling: same parent, next candidate
        const float s2 = __fadd_rn(ns[p], lp[(size_t)(d - 1) * K + j + 1]);
        fk[c] = entry_key(s2, d, p, j + 1, c);
        fs[c] = s2;
        ++c;
      }
      if (kid) {                                        // first child
        const float s3 = __fadd_rn(s, lp[(size_t)d * K]);
        fk[c] = entry_key(s3, d + 1, me, 0, c);
        fs[c] = s3;
      }
    }
    cnt += (sib ? 1 : 0) + (kid ? 1 : 0) - 1;
    __syncwarp();
  }
}

}  // namespace kd

using namespace kd;

extern "C" int kd_tree_build(const float* logp, const int32_t* cand_tokens, const int32_t* root_tokens,
                             int B, int D, int K, int n, int32_t* parents, int32_t* tokens,
                             int32_t* depth, float* score, cudaStream_t stream) {
  if (!logp || !cand_tokens || !root_tokens || !parents || !tokens || !shapes_ok(B, n) || D < 1 ||
      D > 4096 || K < 1 || K > 255)
    return KD_EINVAL;
  // the candidates must hold at least n - 1 nodes: sum over d = 1..D of K^d
  int64_t total = 0, level = 1;
  for (int d = 1; d <= D && total < n - 1; ++d) {
    level = level * K > (int64_t)KD_MAX_NODES ? (int64_t)KD_MAX_NODES : level * K;
    total += level;
  }
  if (total < n - 1) return KD_EINVAL;
  int st = device_sms(nullptr);
  if (st) return st;
  tree_build_kernel<<<(B + TB_WARPS - 1) / TB_WARPS, 32 * TB_WARPS, 0, stream>>>(
      logp, cand_tokens, root_tokens, B, D, K, n, parents, tokens, depth, score);
  return launch_status("tree_build_kernel");
}
