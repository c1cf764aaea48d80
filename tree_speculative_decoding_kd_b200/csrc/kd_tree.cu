// Tree and cache kernels of the verify step: ancestor masks, greedy acceptance,
// node-latent write and post-accept compaction.  All are launch-latency-sized;
// they are written for coalesced 16-byte traffic and warp-level decisions.
//
// Sources (page title, section):
//   "The Architecture of Pragmatic Ambition" -- "The Knowledge Architecture":
//       visibility-masked tree attention; greedy walk to the longest prefix that
//       matches the target's predictions.
//   "The Architectural Keystone: Writing the Model Header ..." -- "The Reasoning
//       That Preceded the Header": budget+1 nodes, root at the next free slot,
//       accepted latents (root included) gathered into contiguous slots and the
//       cache length advanced by the accepted count; "Mistakes and Iterative
//       Refinement": source and destination slots of the gather can overlap, so
//       every kept row is read before any is written.

#include <string.h>

#include "kd_common.cuh"
#include "kd_accept.cuh"

namespace kd {

// ------------------------------------------------------------------ host helpers
static thread_local char g_cuda_err[256];

void set_cuda_error(cudaError_t e, const char* where) {
  snprintf(g_cuda_err, sizeof(g_cuda_err), "%s: %s", where, cudaGetErrorString(e));
}

int device_sms(int* sms) {
  static int cached_major[64], cached_sms[64];
  int dev = 0;
  int st = cuda_status(cudaGetDevice(&dev), "cudaGetDevice");
  if (st) return st;
  if (dev < 0 || dev >= 64) return KD_ENODEV;
  if (cached_major[dev] == 0) {
    int major = 0, count = 0;
    st = cuda_status(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev), "attr");
    if (st) return st;
    st = cuda_status(cudaDeviceGetAttribute(&count, cudaDevAttrMultiProcessorCount, dev), "attr");
    if (st) return st;
    cached_sms[dev] = count;
    cached_major[dev] = major;
  }
  if (cached_major[dev] != 10) return KD_ENODEV;
  if (sms) *sms = cached_sms[dev];
  return KD_OK;
}

// ------------------------------------------------------------------ mask build
// One CTA per request, one thread per node.  A node's mask is the OR of the bits
// of the nodes met walking parent links from it to the root.
__global__ void __launch_bounds__(KD_MAX_NODES)
build_mask_kernel(const int32_t* __restrict__ parents, int n, uint32_t* __restrict__ vis,
                  int32_t* __restrict__ depth, int32_t* dev_error) {
  __shared__ int par[KD_MAX_NODES];
  const int b = blockIdx.x, i = threadIdx.x;
  const int W = (n + 31) >> 5;
  int p = 0;
  bool bad = false;
  if (i < n) {
    p = parents[(size_t)b * n + i];
    bad = (i == 0) ? (p != -1) : (p < 0 || p >= i);
    par[i] = p;
  }
  bad = __syncthreads_or(bad);
  if (i >= n) return;
  uint32_t w[4] = {0u, 0u, 0u, 0u};
  int d = 0;
  if (!bad) {
    int k = i;
    while (k > 0) {             // parent < child, so at most i steps
      w[k >> 5] |= 1u << (k & 31);
      k = par[k];
      ++d;
    }
    w[0] |= 1u;                 // the root is visible to every node
  } else if (i == 0) {
    raise_dev_error(dev_error, KD_DEV_BAD_PARENT);
  }
  uint32_t* row = vis + ((size_t)b * n + i) * W;
  for (int q = 0; q < W; ++q) row[q] = w[q];
  if (depth) depth[(size_t)b * n + i] = d;
}

// ------------------------------------------------------------------ greedy accept
// One warp per request (the walk itself is in kd_accept.cuh).
__global__ void __launch_bounds__(128)
accept_kernel(const int32_t* __restrict__ tokens, const int32_t* __restrict__ parents,
              const int32_t* __restrict__ argmax, int B, int n, int32_t* __restrict__ path,
              int32_t* __restrict__ len, int32_t* __restrict__ bonus, int32_t* dev_error) {
  const int b = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (b >= B) return;
  accept_walk(tokens, parents, argmax, b, n, path, len, bonus, dev_error);
}

// ------------------------------------------------------------------ slot -> cache row
// A request's logical slot s lives in cache row b * cap + s (contiguous caches) or in
// row page_table[b][s / P] * P + s % P of a shared page pool (paged caches: page size
// P > 1, the remedy for the page-size-1 fragmentation of "The Architectural Keystone",
// "Assumptions Embedded in the Design").
struct SlotMap {
  const int32_t* pt;          // [B][M] physical page ids, or nullptr for a contiguous cache
  int64_t cap;                // logical slots per request
  int64_t pages;              // pages in the pool (paged)
  int P, M;                   // page size, pages per request (paged)
  __device__ int64_t row(int b, int64_t s) const {
    return pt ? (int64_t)pt[(size_t)b * M + s / P] * P + s % P : (int64_t)b * cap + s;
  }
  // every page holding slots [s0, s1) is inside the pool (always true when contiguous)
  __device__ bool pages_ok(int b, int64_t s0, int64_t s1) const {
    if (!pt) return true;
    for (int64_t q = s0 / P; q <= (s1 - 1) / P; ++q) {
      const int32_t v = pt[(size_t)b * M + q];
      if (v < 0 || v >= pages) return false;
    }
    return true;
  }
};

// ------------------------------------------------------------------ node write
// One CTA per request; 16-byte copies of the n node rows into slots L..L+n-1.
__global__ void __launch_bounds__(256)
write_nodes_kernel(uint4* __restrict__ c_kv, uint4* __restrict__ k_rope, int64_t sc16,
                   int64_t sr16, SlotMap map, const int32_t* __restrict__ cache_lens,
                   const uint4* __restrict__ node_ckv, const uint4* __restrict__ node_krope,
                   int n, int32_t* dev_error) {
  const int b = blockIdx.x;
  const int64_t L = cache_lens[b];
  if (L < 0 || L + n > map.cap) {
    if (threadIdx.x == 0) raise_dev_error(dev_error, KD_DEV_CACHE_FULL);
    return;
  }
  if (!map.pages_ok(b, L, L + n)) {
    if (threadIdx.x == 0) raise_dev_error(dev_error, KD_DEV_BAD_PAGE);
    return;
  }
  constexpr int CC = KD_D_C / 8, CR = KD_D_R / 8;   // uint4 per row
  for (int idx = threadIdx.x; idx < n * (CC + CR); idx += blockDim.x) {
    const int k = idx / (CC + CR), q = idx % (CC + CR);
    const int64_t r = map.row(b, L + k);
    if (q < CC)
      c_kv[r * sc16 + q] = node_ckv[((size_t)b * n + k) * CC + q];
    else
      k_rope[r * sr16 + (q - CC)] = node_krope[((size_t)b * n + k) * CR + (q - CC)];
  }
}

// ------------------------------------------------------------------ compaction
// One CTA per request.  Phase 1 reads every row that moves (path[j] != j) into
// shared memory; phase 2 writes them to slots L+j.  Rows with path[j] == j are
// already in place.  Shared memory holds up to n rows of 1152 bytes.
__global__ void __launch_bounds__(256)
compact_kernel(uint4* __restrict__ c_kv, uint4* __restrict__ k_rope, int64_t sc16, int64_t sr16,
               SlotMap map, const int32_t* __restrict__ path, const int32_t* __restrict__ len,
               int32_t* __restrict__ cache_lens, int n, int32_t* dev_error) {
  extern __shared__ uint4 stage[];
  __shared__ int src[KD_MAX_NODES], dst[KD_MAX_NODES];
  __shared__ int moves, ok;
  constexpr int CC = KD_D_C / 8, CR = KD_D_R / 8, ROW = CC + CR;
  const int b = blockIdx.x;
  const int64_t L = cache_lens[b];
  const int m = len[b];
  if (threadIdx.x == 0) {
    int good = 1, err = 0;
    if (m < 1 || m > n) { good = 0; err |= KD_DEV_BAD_PATH; }
    if (L < 0 || L + n > map.cap) { good = 0; err |= KD_DEV_CACHE_FULL; }
    else if (!map.pages_ok(b, L, L + n)) { good = 0; err |= KD_DEV_BAD_PAGE; }
    int c = 0;
    for (int j = 0; good && j < m; ++j) {
      const int p = path[(size_t)b * n + j];
      if (p < 0 || p >= n) { good = 0; err |= KD_DEV_BAD_PATH; break; }
      if (p != j) { src[c] = p; dst[c] = j; ++c; }
    }
    moves = c;
    ok = good;
    if (err) raise_dev_error(dev_error, err);
  }
  __syncthreads();
  if (!ok) return;
  const int total = moves * ROW;
  for (int idx = threadIdx.x; idx < total; idx += blockDim.x) {      // read all ...
    const int r = idx / ROW, q = idx % ROW;
    const int64_t s = map.row(b, L + src[r]);
    stage[idx] = (q < CC) ? c_kv[s * sc16 + q] : k_rope[s * sr16 + (q - CC)];
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < total; idx += blockDim.x) {      // ... then write
    const int r = idx / ROW, q = idx % ROW;
    const int64_t d = map.row(b, L + dst[r]);
    if (q < CC) c_kv[d * sc16 + q] = stage[idx];
    else k_rope[d * sr16 + (q - CC)] = stage[idx];
  }
  if (threadIdx.x == 0) cache_lens[b] = (int32_t)(L + m);
}

}  // namespace kd

using namespace kd;

// ================================================================== C ABI
extern "C" int kd_tree_build_mask(const int32_t* parents, int B, int n, uint32_t* vis,
                                  int32_t* depth, int32_t* dev_error, cudaStream_t stream) {
  if (!parents || !vis || !shapes_ok(B, n)) return KD_EINVAL;
  int st = device_sms(nullptr);
  if (st) return st;
  build_mask_kernel<<<B, KD_MAX_NODES, 0, stream>>>(parents, n, vis, depth, dev_error);
  return launch_status("build_mask_kernel");
}

extern "C" int kd_tree_accept(const int32_t* node_tokens, const int32_t* parents,
                              const int32_t* target_argmax, int B, int n, int32_t* path,
                              int32_t* len, int32_t* bonus, int32_t* dev_error,
                              cudaStream_t stream) {
  if (!node_tokens || !parents || !target_argmax || !path || !len || !bonus || !shapes_ok(B, n))
    return KD_EINVAL;
  int st = device_sms(nullptr);
  if (st) return st;
  const int per_cta = 4;
  accept_kernel<<<(B + per_cta - 1) / per_cta, 32 * per_cta, 0, stream>>>(
      node_tokens, parents, target_argmax, B, n, path, len, bonus, dev_error);
  return launch_status("accept_kernel");
}

extern "C" int kd_kv_write_nodes(kd_bf16_t* c_kv, kd_bf16_t* k_rope, int64_t sc, int64_t sr,
                                 int64_t cap, const int32_t* cache_lens, const kd_bf16_t* node_ckv,
                                 const kd_bf16_t* node_krope, int B, int n, int32_t* dev_error,
                                 cudaStream_t stream) {
  if (!cache_ok(c_kv, k_rope, sc, sr, cap) || !cache_lens || !node_ckv || !node_krope ||
      !aligned16(node_ckv) || !aligned16(node_krope) || !shapes_ok(B, n))
    return KD_EINVAL;
  int st = device_sms(nullptr);
  if (st) return st;
  const SlotMap map{nullptr, cap, 0, 1, 0};
  write_nodes_kernel<<<B, 256, 0, stream>>>(
      reinterpret_cast<uint4*>(c_kv), reinterpret_cast<uint4*>(k_rope), sc / 8, sr / 8, map,
      cache_lens, reinterpret_cast<const uint4*>(node_ckv),
      reinterpret_cast<const uint4*>(node_krope), n, dev_error);
  return launch_status("write_nodes_kernel");
}

static bool paged_ok(const int32_t* page_table, int page_size, int64_t pages_per_req, int64_t num_pages) {
  return page_table && page_size >= 1 && pages_per_req >= 1 && num_pages >= 1 &&
         num_pages * page_size <= (int64_t)INT32_MAX && pages_per_req * page_size <= (int64_t)INT32_MAX;
}

extern "C" int kd_kv_write_nodes_paged(kd_bf16_t* c_pages, kd_bf16_t* r_pages, int64_t sc, int64_t sr,
                                       int page_size, const int32_t* page_table, int64_t pages_per_req,
                                       int64_t num_pages, const int32_t* cache_lens,
                                       const kd_bf16_t* node_ckv, const kd_bf16_t* node_krope, int B,
                                       int n, int32_t* dev_error, cudaStream_t stream) {
  if (!paged_ok(page_table, page_size, pages_per_req, num_pages) ||
      !cache_ok(c_pages, r_pages, sc, sr, num_pages * page_size) || !cache_lens || !node_ckv ||
      !node_krope || !aligned16(node_ckv) || !aligned16(node_krope) || !shapes_ok(B, n))
    return KD_EINVAL;
  int st = device_sms(nullptr);
  if (st) return st;
  const SlotMap map{page_table, pages_per_req * page_size, num_pages, page_size, (int)pages_per_req};
  write_nodes_kernel<<<B, 256, 0, stream>>>(
      reinterpret_cast<uint4*>(c_pages), reinterpret_cast<uint4*>(r_pages), sc / 8, sr / 8, map,
      cache_lens, reinterpret_cast<const uint4*>(node_ckv),
      reinterpret_cast<const uint4*>(node_krope), n, dev_error);
  return launch_status("write_nodes_kernel");
}

// Device check plus the compaction kernel's shared-memory limit (once per device).
static int compact_setup() {
  int st = device_sms(nullptr);
  if (st) return st;
  static bool attr_set[64];
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    st = cuda_status(cudaFuncSetAttribute(compact_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          KD_MAX_NODES * (KD_D_C + KD_D_R) * 2),
                     "cudaFuncSetAttribute(compact_kernel)");
    if (st) return st;
    attr_set[dev] = true;
  }
  return KD_OK;
}

extern "C" int kd_kv_compact(kd_bf16_t* c_kv, kd_bf16_t* k_rope, int64_t sc, int64_t sr,
                             int64_t cap, const int32_t* path, const int32_t* len,
                             int32_t* cache_lens, int B, int n, int32_t* dev_error,
                             cudaStream_t stream) {
  if (!cache_ok(c_kv, k_rope, sc, sr, cap) || !path || !len || !cache_lens || !shapes_ok(B, n))
    return KD_EINVAL;
  int st = compact_setup();
  if (st) return st;
  const size_t smem = (size_t)n * (KD_D_C + KD_D_R) * 2;
  const SlotMap map{nullptr, cap, 0, 1, 0};
  compact_kernel<<<B, 256, smem, stream>>>(reinterpret_cast<uint4*>(c_kv),
                                           reinterpret_cast<uint4*>(k_rope), sc / 8, sr / 8, map,
                                           path, len, cache_lens, n, dev_error);
  return launch_status("compact_kernel");
}

extern "C" int kd_kv_compact_paged(kd_bf16_t* c_pages, kd_bf16_t* r_pages, int64_t sc, int64_t sr,
                                   int page_size, const int32_t* page_table, int64_t pages_per_req,
                                   int64_t num_pages, const int32_t* path, const int32_t* len,
                                   int32_t* cache_lens, int B, int n, int32_t* dev_error,
                                   cudaStream_t stream) {
  if (!paged_ok(page_table, page_size, pages_per_req, num_pages) ||
      !cache_ok(c_pages, r_pages, sc, sr, num_pages * page_size) || !path || !len || !cache_lens ||
      !shapes_ok(B, n))
    return KD_EINVAL;
  int st = compact_setup();
  if (st) return st;
  const size_t smem = (size_t)n * (KD_D_C + KD_D_R) * 2;
  const SlotMap map{page_table, pages_per_req * page_size, num_pages, page_size, (int)pages_per_req};
  compact_kernel<<<B, 256, smem, stream>>>(reinterpret_cast<uint4*>(c_pages),
                                           reinterpret_cast<uint4*>(r_pages), sc / 8, sr / 8, map,
                                           path, len, cache_lens, n, dev_error);
  return launch_status("compact_kernel");
}

extern "C" int kd_read_device_error(int32_t* dev_error, int clear, cudaStream_t stream) {
  if (!dev_error) return KD_EINVAL;
  int32_t v = 0;
  int st = cuda_status(cudaMemcpyAsync(&v, dev_error, sizeof(v), cudaMemcpyDeviceToHost, stream),
                       "cudaMemcpyAsync(error word)");
  if (st) return st;
  if (clear) {
    st = cuda_status(cudaMemsetAsync(dev_error, 0, sizeof(int32_t), stream), "cudaMemsetAsync");
    if (st) return st;
  }
  st = cuda_status(cudaStreamSynchronize(stream), "cudaStreamSynchronize");
  if (st) return st;
  return v;
}

extern "C" const char* kd_strerror(int code) {
  switch (code) {
    case KD_OK: return "ok";
    case KD_EINVAL: return "invalid argument (null pointer, shape, limit or alignment)";
    case KD_ERANGE: return "workspace too small or size beyond the supported maximum";
    case KD_ELAUNCH: return g_cuda_err[0] ? g_cuda_err : "CUDA error";
    case KD_ENODEV: return "current device is not an sm_100 (B200-class) GPU";
    default: return "unknown kd error code";
  }
}
