// Greedy acceptance of one verified tree by one warp ("The Architecture of
// Pragmatic Ambition", section "The Knowledge Architecture": walk the tree to the
// longest prefix that matches the target's predictions).  Shared by the plain
// accept kernel and the one fused with the target argmax.
#pragma once

#include "kd_common.cuh"

namespace kd {

// Lane l holds nodes l, l+32, l+64, l+96.  Each step is one ballot per 32-node
// chunk; the first chunk with a match gives the lowest-index matching child.
// All 32 lanes of the warp call it for request b; argmax may be written by this warp
// just before (it is read back through the same SM).
__device__ __forceinline__ void accept_walk(const int32_t* __restrict__ tokens,
                                            const int32_t* __restrict__ parents,
                                            const int32_t* argmax, int b, int n,
                                            int32_t* __restrict__ path, int32_t* __restrict__ len,
                                            int32_t* __restrict__ bonus, int32_t* dev_error) {
  const int lane = threadIdx.x & 31;
  const size_t base = (size_t)b * n;
  int par[4], tok[4];
  bool bad = false;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const int node = c * 32 + lane;
    par[c] = -2;
    tok[c] = 0;
    if (node < n) {
      par[c] = parents[base + node];
      tok[c] = tokens[base + node];
      bad |= (node == 0) ? (par[c] != -1) : (par[c] < 0 || par[c] >= node);
    }
  }
  bad = __any_sync(0xffffffffu, bad);
  int cur = 0, cnt = 1;
  if (lane == 0) path[base] = 0;
  if (bad) {
    if (lane == 0) raise_dev_error(dev_error, KD_DEV_BAD_PARENT);
  } else {
    while (cnt < n) {
      const int want = argmax[base + cur];
      int next = -1;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const unsigned m = __ballot_sync(0xffffffffu, par[c] == cur && tok[c] == want);
        if (next < 0 && m) next = c * 32 + __ffs(m) - 1;
      }
      if (next < 0) break;
      cur = next;
      if (lane == 0) path[base + cnt] = cur;
      ++cnt;
    }
  }
  for (int j = cnt + lane; j < n; j += 32) path[base + j] = -1;
  if (lane == 0) {
    len[b] = cnt;
    bonus[b] = argmax[base + cur];
  }
}

}  // namespace kd
