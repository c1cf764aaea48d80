// Delivery probes of the trace build (libkdverify_trace.so only; the product library
// does not contain this file).
//
// How many bytes per SM cycle TMA tile loads deliver from an L2-resident window when a
// ring of `depth` boxes is kept in flight, issued and waited on the way the attention's
// K ring is (one thread issues; a stage is reused once its previous load landed; waits
// poll the barrier and read the global timer once per 64 polls):
//   - kd_probe_l2_boxes, pair = 0: one CTA per SM, each loading whole boxes;
//   - pair = 1: 2-CTA clusters whose CTAs each load half of every box into their own
//     shared memory, both halves completing on the even CTA's barrier (the load form a
//     pair-MMA design would use for its B operand: cta_group::2, no multicast); the
//     even CTA hands each stage back to the odd one with a remote arrive.
// Every wait is bounded (2 s); one that gives up sets *err and the CTA drains and exits.
//
// kd_probe_store measures the other direction, in the attention epilogue's pattern: each CTA
// writes a 128 x 512 fp32 tile (256 KB, one split partial) into its own plane, `reps` times
// back to back, and waits once at the end for every store to complete:
//   - mode 0: 8 warps, lane 0 of each issuing 2 KB TMA box stores (16 columns x 32 rows,
//     64-byte swizzle) from its staging slot, as the epilogue does;
//   - mode 1: the same in 4 KB boxes (32 columns x 32 rows, 128-byte swizzle);
//   - mode 2: plain 16-byte stores from 256 threads, each warp instruction writing 512
//     contiguous bytes of a row.
//
// kd_probe_mma measures the tensor pipe as its issuing threads see it: each CTA (one per SM)
// issues `count` tcgen05.mma (kind::f16, bf16, M = 64 or 128, K = 16, N = 64 / 128 / 256) back to back
// from one thread (or from two threads in two warps, each into its own accumulator) into TMEM,
// A from shared memory or from TMEM, B from shared memory, and with
// `wait_every` > 0 it polls an already-completed mbarrier after every `wait_every` MMAs (a
// shared-memory read while MMAs are in flight, as a pipeline's per-stage wait is).  One commit
// at the end; the cycles run from the first issue to that commit's arrival.

#include <cuda.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <mutex>

#include "kd_common.cuh"
#include "kd_ptx.cuh"

namespace kd {
namespace probe {

using namespace ptx;

constexpr int MAX_DEPTH = 24;
constexpr uint64_t LIMIT_NS = 2000000000ull;

__device__ __forceinline__ bool poll(uint32_t bar, uint32_t parity, bool cluster_scope) {
  uint64_t t0 = 0;
  for (uint32_t spin = 0;; ++spin) {
    if (cluster_scope ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity)) return true;
    if ((spin & 63u) == 63u) {
      const uint64_t t = globaltimer();
      if (t0 == 0) t0 = t;
      else if (t - t0 > LIMIT_NS) return false;
    }
  }
}

// The pair form of the tiled load: the destination is this CTA's shared memory, the
// barrier may be the peer's (cluster address).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const void* map, int32_t x, int32_t y,
                                                 uint32_t bar_cluster) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar_cluster)
      : "memory");
}

// Shared memory: FULL barriers at base, EMPTY barriers at base + 256, stages from
// base + 1024 (1024-byte aligned, `stage_bytes` apart).
// With `issuers` warps, warp w's lane 0 runs its own ring of depth / issuers stages
// (its own barriers, stages and rows), so the CTA keeps `depth` boxes in flight either way.
__global__ void __launch_bounds__(64, 1)
l2_box_kernel(const __grid_constant__ CUtensorMap tm, int box_rows, int depth, int iters, int window_rows,
              unsigned long long* cycles, int* err) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t stage_bytes = (uint32_t)box_rows * 128u;
  const int issuers = blockDim.x / 32, w = threadIdx.x >> 5;
  const int all_stages = depth;
  depth /= issuers;
  const uint32_t base0 = (raw + 1023u) & ~1023u;
  if (threadIdx.x == 0) {
    for (int s = 0; s < all_stages; ++s) mbar_init(base0 + 8u * s, 1);
    fence_mbar_init();
  }
  __syncthreads();
  // warp w: barriers from base0 + 8 (w depth), stages from base0 + 1024 + w depth stage_bytes
  const uint32_t base = base0 + 8u * w * depth;
  const uint32_t stages = base0 + 1024u + (uint32_t)(w * depth) * stage_bytes;
  if ((threadIdx.x & 31) == 0) {
    // no division in the loop: the row advances by one box and wraps; stage s and the
    // parity of its next completion are counters
    int y = (int)(((long long)(blockIdx.x * issuers + w) * 7919 * box_rows) % window_rows);
    bool ok = true;
    uint32_t par = 0;                        // parity of stage s's next completion, bit per stage
    const long long t0 = clock64();
    int i = 0, s = 0;
    for (; i < iters && ok; ++i) {
      if (i >= depth) {
        if (!(ok = poll(base + 8u * s, (par >> s) & 1u, false))) break;
        par ^= 1u << s;
      }
      mbar_arrive_expect_tx(base + 8u * s, stage_bytes);
      tma_load_2d(stages + s * stage_bytes, &tm, 0, y, base + 8u * s);
      y += box_rows;
      if (y >= window_rows) y -= window_rows;
      if (++s == depth) s = 0;
    }
    for (int j = 0; j < depth && j < i; ++j) {     // the last loads, in issue order from stage s
      if (!poll(base + 8u * s, (par >> s) & 1u, false)) ok = false;
      par ^= 1u << s;
      if (++s == depth) s = 0;
    }
    atomicMax(cycles + blockIdx.x, (unsigned long long)(clock64() - t0));
    if (!ok) atomicOr(err, 1);
  }
  __syncthreads();
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(32, 1)
l2_pair_kernel(const __grid_constant__ CUtensorMap tm, int box_rows, int depth, int iters, int window_rows,
               unsigned long long* cycles, int* err) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  const uint32_t rank = cluster_ctarank();
  const uint32_t half_rows = (uint32_t)box_rows / 2;
  const uint32_t stage_bytes = half_rows * 128u;
  if (threadIdx.x == 0) {
    for (int s = 0; s < depth; ++s) {
      mbar_init(base + 8u * s, 1);          // FULL (used in the even CTA)
      mbar_init(base + 256u + 8u * s, 1);   // EMPTY (used in the odd CTA)
    }
    fence_mbar_init();
  }
  cluster_sync();
  const uint32_t full_even = map_to_rank(base, 0);        // FULL barriers of the even CTA
  const uint32_t empty_odd = map_to_rank(base + 256u, 1);   // EMPTY barriers of the odd CTA
  if (threadIdx.x == 0) {
    int y = (int)(((long long)(blockIdx.x / 2) * 7919 * box_rows) % window_rows);
    bool ok = true;
    uint32_t par = 0;
    const long long t0 = clock64();
    int i = 0, s = 0;
    for (; i < iters && ok; ++i) {
      if (rank == 0) {
        if (i >= depth) {
          if (!(ok = poll(base + 8u * s, (par >> s) & 1u, true))) break;
          mbar_arrive_remote(empty_odd + 8u * s);                 // the odd CTA may reuse stage s
        }
        mbar_arrive_expect_tx(base + 8u * s, 2u * stage_bytes);
      } else if (i >= depth && !(ok = poll(base + 256u + 8u * s, (par >> s) & 1u, true))) {
        break;
      }
      if (i >= depth) par ^= 1u << s;
      tma_load_2d_pair(base + 1024u + s * stage_bytes, &tm, 0, y + (int)(rank * half_rows), full_even + 8u * s);
      y += box_rows;
      if (y >= window_rows) y -= window_rows;
      if (++s == depth) s = 0;
    }
    // the even CTA waits for the last loads and releases their stages; the odd CTA
    // waits for those releases, so neither leaves with a load in flight
    for (int j = 0; j < depth && j < i; ++j) {
      if (rank == 0) {
        if (!poll(base + 8u * s, (par >> s) & 1u, true)) ok = false;
        mbar_arrive_remote(empty_odd + 8u * s);
      } else if (!poll(base + 256u + 8u * s, (par >> s) & 1u, true)) {
        ok = false;
      }
      par ^= 1u << s;
      if (++s == depth) s = 0;
    }
    cycles[blockIdx.x] = (unsigned long long)(clock64() - t0);
    if (!ok) atomicOr(err, 1);
  }
  __syncwarp();
  cluster_sync();
}

// Shared memory: eight 4 KB staging slots (one per warp) from a 1024-byte aligned base; their
// content is irrelevant and never rewritten, so a slot is reused without waiting for reads.
__global__ void __launch_bounds__(256, 1)
store_kernel(const __grid_constant__ CUtensorMap tm, float* buf, int mode, int reps, unsigned long long* cycles) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < 8 * 4096 / 16; i += 256) st_shared_v4(base + i * 16, 0u, 0u, 0u, 0u);
  fence_proxy_async_cta();
  __syncthreads();
  const long long t0 = clock64();
  const int z = blockIdx.x;
  const int row0 = (warp & 3) * 32, col0 = (warp >> 2) * 256;   // the warp's 32 rows x 256 columns
  if (mode < 2) {
    if (lane == 0) {
      const int w = mode == 0 ? 16 : 32;                           // columns per box
      for (int rep = 0; rep < reps; ++rep)
        for (int c = 0; c < 256 / w; ++c) {
          tma_store_3d(&tm, base + warp * 4096, col0 + c * w, row0, z);
          bulk_commit_group();
        }
      bulk_wait_group0();
    }
    __syncwarp();
  } else {
    float* dst = buf + ((size_t)z * 128 + row0) * 512 + col0;
    for (int rep = 0; rep < reps; ++rep)
      for (int rr = 0; rr < 32; ++rr) {
        st_global_v4(dst + rr * 512 + lane * 4, 0u, 0u, 0u, 0u);
        st_global_v4(dst + rr * 512 + 128 + lane * 4, 0u, 0u, 0u, 0u);
      }
    __threadfence();
  }
  __syncthreads();
  if (threadIdx.x == 0) cycles[blockIdx.x] = (unsigned long long)(clock64() - t0);
}

// Shared memory from a 1024-byte aligned base: TMEM address at +0, barriers at +64 and +80
// (done, one per issuer) and +72 (ready), A (128 rows x 64 bf16, 16 KB) at +1024, B (256 rows x 64 bf16, 32 KB) at
// +17408; both zero, 128-byte swizzled K-major.  The dynamic size (> half an SM's) keeps one
// CTA per SM, so the 512-column allocation never waits for another CTA.
constexpr int MMA_SMEM = 120 * 1024;
template <bool A_TMEM>
__global__ void __launch_bounds__(128, 1)
mma_kernel(int m, int n, int issuers, int count, int wait_every, unsigned long long* cycles, int* err) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const int warp = threadIdx.x >> 5;
  const uint32_t done = base + 64, ready = base + 72, a_s = base + 1024, b_s = base + 1024 + 16384;
  for (int i = threadIdx.x; i < (16384 + 32768) / 16; i += 128) st_shared_v4(a_s + i * 16, 0u, 0u, 0u, 0u);
  if (threadIdx.x == 0) {
    mbar_init(done, 1);
    mbar_init(done + 16, 1);
    mbar_init(ready, 1);
    fence_mbar_init();
    mbar_arrive(ready);                  // phase 0 of `ready` is complete from the start
  }
  fence_proxy_async_cta();
  if (warp == 0) {
    tmem_alloc(base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem_raw + (base - smem_u32(smem_raw)));
  // issuer w (lane 0 of warp w < issuers) accumulates into TMEM columns [w n, (w + 1) n), takes
  // A from TMEM columns 256 + 128 w on (or from the shared A tile, which both only read), and
  // issues count / issuers MMAs
  const int lane = threadIdx.x & 31;
  if (lane == 0 && warp < issuers) {
    const uint32_t idesc = ((1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) |
                            ((uint32_t)(m >> 4) << 24));
    const uint32_t d = tmem + (uint32_t)(warp * n), a_t = tmem + 256 + warp * 128;
    // descriptors formed before the clock starts; 4 MMAs (one 64-column K chunk) per loop
    // trip, and the wait cadence kept by a countdown rather than a division
    uint64_t ad[4], bd[4];
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      ad[kk] = smem_desc_sw128(a_s + kk * 32, 16, 1024);
      bd[kk] = smem_desc_sw128(b_s + kk * 32, 16, 1024);
    }
    const int mine = count / issuers;
    const uint32_t bar = done + 16u * warp;
    int left = wait_every;
    const long long t0 = clock64();
    for (int i = 0; i < mine; i += 4) {
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint32_t acc = (i | kk) != 0 ? 1u : 0u;
        if (A_TMEM) mma_bf16_ts(d, a_t + kk * 8, bd[kk], idesc, acc);
        else mma_bf16_ss(d, ad[kk], bd[kk], idesc, acc);
      }
      if (wait_every > 0 && (left -= 4) <= 0) {
        (void)mbar_try_wait(ready, 0);
        left = wait_every;
      }
    }
    tc_commit(bar);
    bool ok = poll(bar, 0, false);
    const long long t1 = clock64();
    if (!ok) {                           // MMAs always finish: wait again (bounded) before freeing TMEM
      atomicOr(err, 1);
      poll(bar, 0, false);
    }
    atomicMax(cycles + blockIdx.x, (unsigned long long)(t1 - t0));
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static std::once_flag once;
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

}  // namespace probe
}  // namespace kd

// buf: bf16 [rows][512] on the device (rows a multiple of box_rows); box_rows 32..256 (even),
// depth 1..24 boxes in flight, pair 0 or 1.  cycles: device uint64 [grid CTAs]; err: device
// int32 (ORed).  Grid: 148 CTAs (74 clusters when pair).
extern "C" int kd_probe_l2_boxes(const void* buf, int rows, int box_rows, int depth, int iters, int pair,
                                 unsigned long long* cycles, int* err, cudaStream_t stream) {
  // pair: 0 whole boxes, one issuing warp; 1 pair loads; 2 whole boxes, two issuing warps
  const int issuers = pair == 2 ? 2 : 1;
  if (pair == 2) pair = 0;
  if (depth % issuers) return KD_EINVAL;
  using namespace kd::probe;
  if (!buf || !cycles || !err || box_rows < 32 || box_rows > 256 || (box_rows & 1) || depth < 1 ||
      depth > MAX_DEPTH || iters < depth || rows < box_rows || rows % box_rows)
    return KD_EINVAL;
  const size_t smem = 1024 + 1024 + (size_t)depth * box_rows * 128 / (pair ? 2 : 1);
  if (smem > 232448) return KD_ERANGE;
  auto fn = encode_fn();
  if (!fn) return KD_ELAUNCH;
  CUtensorMap tm;
  cuuint64_t dims[2] = {512, (cuuint64_t)rows};
  cuuint64_t strides[1] = {1024};
  cuuint32_t box[2] = {64, (cuuint32_t)(pair ? box_rows / 2 : box_rows)};
  cuuint32_t es[2] = {1, 1};
  if (fn(&tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(buf), dims, strides, box, es,
         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return KD_ELAUNCH;
  int st;
  if (pair) {
    if ((st = kd::cuda_status(cudaFuncSetAttribute(l2_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   (int)smem), "cudaFuncSetAttribute(probe)")))
      return st;
    l2_pair_kernel<<<148, 32, smem, stream>>>(tm, box_rows, depth, iters, rows, cycles, err);
  } else {
    if ((st = kd::cuda_status(cudaFuncSetAttribute(l2_box_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   (int)smem), "cudaFuncSetAttribute(probe)")))
      return st;
    l2_box_kernel<<<148, 32 * issuers, smem, stream>>>(tm, box_rows, depth, iters / issuers, rows, cycles, err);
  }
  return kd::launch_status("l2 probe");
}

// buf: device fp32 [ctas][128][512]; ctas 1..148; mode 0..2; reps >= 1.  cycles: device uint64
// [ctas] (SM cycles from the first store to the last completion, per CTA).
extern "C" int kd_probe_store(void* buf, int ctas, int mode, int reps, unsigned long long* cycles,
                              cudaStream_t stream) {
  using namespace kd::probe;
  if (!buf || !cycles || ctas < 1 || ctas > 148 || mode < 0 || mode > 2 || reps < 1) return KD_EINVAL;
  auto fn = encode_fn();
  if (!fn) return KD_ELAUNCH;
  CUtensorMap tm;
  const int w = mode == 1 ? 32 : 16;
  cuuint64_t dims[3] = {512, 128, (cuuint64_t)ctas};
  cuuint64_t strides[2] = {512 * 4, 128 * 512 * 4};
  cuuint32_t box[3] = {(cuuint32_t)w, 32, 1};
  cuuint32_t es[3] = {1, 1, 1};
  if (fn(&tm, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, buf, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
         mode == 1 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return KD_ELAUNCH;
  const int smem = 8 * 4096 + 1024;
  int st;
  if ((st = kd::cuda_status(cudaFuncSetAttribute(store_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem),
                            "cudaFuncSetAttribute(store probe)")))
    return st;
  store_kernel<<<ctas, 256, smem, stream>>>(tm, static_cast<float*>(buf), mode, reps, cycles);
  return kd::launch_status("store probe");
}

// m in {64, 128} (64 with A from shared memory only); n in {64, 128, 256}; a_tmem 0 / 1; issuers 1,
// or 2 with n <= 128 (each its own accumulator);
// count in [4 issuers, 2^22] and wait_every >= 0, multiples of 4 (count of 4 issuers).  cycles:
// device uint64 [148], zeroed by the caller (the slower issuer's time per CTA); err: device
// int32 (ORed; set if a final wait gave up once).  Grid: 148 CTAs.
extern "C" int kd_probe_mma(int m, int n, int a_tmem, int issuers, int count, int wait_every,
                            unsigned long long* cycles, int* err, cudaStream_t stream) {
  using namespace kd::probe;
  if (!cycles || !err || (m != 64 && m != 128) || (n != 64 && n != 128 && n != 256) || (a_tmem != 0 && a_tmem != 1) ||
      (m == 64 && a_tmem) ||
      (issuers != 1 && issuers != 2) || (issuers == 2 && n > 128) || count < 4 * issuers || count > (1 << 22) ||
      count % (4 * issuers) || wait_every < 0 || (wait_every & 3))
    return KD_EINVAL;
  int st;
  auto kern = a_tmem ? mma_kernel<true> : mma_kernel<false>;
  if ((st = kd::cuda_status(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, MMA_SMEM),
                            "cudaFuncSetAttribute(mma probe)")))
    return st;
  kern<<<148, 128, MMA_SMEM, stream>>>(m, n, issuers, count, wait_every, cycles, err);
  return kd::launch_status("mma probe");
}
