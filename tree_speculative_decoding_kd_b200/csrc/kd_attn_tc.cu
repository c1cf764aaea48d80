// Tree-verify MLA-absorb attention on sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// Definition ("The Architecture of Pragmatic Ambition", "The Thinking Process" --
// absorb form: q_nope . (W_UK c_kv) = (q_nope W_UK) . c_kv -- and "The Knowledge
// Architecture" -- tree attention under a visibility mask; "The Architectural
// Keystone ...", "The Reasoning That Preceded the Header" -- node k of the
// budget+1 tree lives in slot L+k):
//   row (i, h) of request b sees slots [0, L) and {L+k : bit k of vis[b][i]};
//   s = scale (q_abs . c_kv + q_rope . k_rope), out = softmax(s) . c_kv, lse = ln sum exp s.
//
// Because the latent is shared by all heads, a request's n*H query rows against
// its keys form a dense (n*H x 576) . (576 x keys) contraction followed by a
// (n*H x keys) . (keys x 512) one.  Rows are node-major (row = i*H + h) and cut
// into 128-row M tiles; keys are streamed in 256-key QK tiles, each split into two
// 128-key P tiles.
//
// The fp32 output accumulator of one M tile (128 x 512) fills all 512 TMEM
// columns of an SM, leaving none for scores, so each unit of work (request, M tile,
// key partition) runs on a 2-CTA cluster with split roles:
//   rank 0 ("QK" CTA): S = Q K^T for 256 keys at a time (M=128, N=256 MMAs, the
//       shape that keeps the tensor pipe saturated from one issuing thread) into
//       256 TMEM columns.  The eight 64-wide latent chunks of Q sit in the other 256
//       TMEM columns and feed the MMA as its A operand from tensor memory; the rope
//       chunk sits in shared memory.  Shared memory holds a 4-stage ring of
//       256-key x 64-column K chunks (TMA, 128-byte swizzle) and two P staging
//       slots.  Two 4-warp softmax groups copy S into registers (freeing TMEM for
//       the next tile at once), take the row max on raw scores with the
//       three-operand max, keep an online max with a lazy rescale threshold, and
//       emit P as two 128-key halves (scale and reference folded into one packed
//       f32x2 FMA per key pair, sums in packed f32x2 adds): each half is written
//       into a local staging slot in the K-major swizzled layout the MMA reads and
//       moved to rank 1 by one thread with a single bulk copy that completes on
//       rank 1's barrier.
//   rank 1 ("PV" CTA): O (128 x 512 fp32) in TMEM; V as 64-key x 256-column
//       groups (four 64-column MN-major boxes) in a 4-deep ring; O += P V as
//       M=128, N=256, K=16 MMAs; V groups wholly past the request's last key are
//       neither loaded nor multiplied.  Two 4-warp groups apply the rare O rescale
//       and write the normalised bf16 output (or an fp32 split-KV partial) through
//       swizzled shared-memory boxes and TMA stores, 256 columns each.
// QK work (576-deep) and PV work (512-deep) are nearly equal, so the pair keeps
// both tensor pipes busy.  Both CTAs read the same c_kv tile (the second read
// hits L2).  Units go out longest request first.  No TMA multicast is used anywhere.
//
// attn_tc_kernel<true> reads a paged cache instead: each 256-key K stage arrives as
// one TMA box per page and each 64-key V group as one box inside a page, from the
// unit's slice of the page table staged in shared memory; nothing else differs.
//
// Every mbarrier wait is bounded (globaltimer); a wait that gives up raises
// KD_DEV_TIMEOUT, marks both CTAs aborted, and every role falls through to the
// common teardown (cluster barrier, TMEM release).

#include <cuda.h>
#include <cudaTypedefs.h>
#include <math.h>

#include "kd_common.cuh"
#include "kd_ptx.cuh"

namespace kd {

int launch_combine(const float* part_o, const float* part_lse, const int32_t* cache_lens, int B,
                   int n, int H, int64_t cap, int splits, uint16_t* out, float* lse,
                   cudaStream_t stream);

namespace tc {

using namespace ptx;

constexpr int NTHREADS = 320;           // warp 0 TMA, warp 1 MMA, warps 2..9 two 4-warp groups
constexpr int GROUP = 256;              // threads of the two 4-warp groups
constexpr int BM = 128;                 // query rows per M tile
constexpr int BQ = 256;                 // keys per QK tile (S = 128 x 256)
constexpr int BN = 128;                 // keys per P / PV tile (two per QK tile)
constexpr int KC = 64;                  // columns per 128-byte swizzle atom
constexpr int NCHUNK = 9;               // 8 latent chunks + 1 rope chunk
constexpr int CHUNK = BN * KC * 2;      // 16 KB: 128 rows x 64 bf16
constexpr int KCHUNK = BQ * KC * 2;     // 32 KB: 256 keys x 64 bf16 (one K ring stage)
constexpr int NQT = 8;                  // Q chunks held in TMEM (the rope chunk in shared memory)
constexpr int NK = 4;                   // K ring stages
constexpr int VKEYS = 64;               // keys per V group
constexpr int VCH = VKEYS * KC * 2;     // 8 KB: 64 keys x 64 latent columns
constexpr int VG = 4 * VCH;             // one V group: 64 keys x 256 latent columns
constexpr int NVG = 4;                  // V ring depth
constexpr int PBYTES = BM * BN * 2;     // one bf16 P tile (two 16 KB swizzle columns)
constexpr int SLOT_ALPHA = PBYTES;      // f32 [128] per-row rescale factor
constexpr int SLOT_FLAG = PBYTES + 512; // u32 rescale-needed flag
constexpr int SLOT_COPY = PBYTES + 528; // bytes moved to the PV CTA per tile
constexpr int PSLOT = PBYTES + 1024;    // slot stride (keeps 1024-byte alignment)

// TMEM columns of the QK CTA
constexpr uint32_t TS = 0;              // S: 256 columns (one 128 x 256 tile)
constexpr uint32_t TQ = 256;            // Q chunks 0..7: 8 x 32 columns

// control block (same offsets in both CTAs so the peer can address it)
constexpr int CTRL = 4096;
enum Bar {
  Q_FULL = 0,
  QT_FULL = Q_FULL + 1,
  K_FULL = QT_FULL + 1,
  K_EMPTY = K_FULL + NK,
  S_FULL = K_EMPTY + NK,
  S_EMPTY = S_FULL + 1,
  P_FREE = S_EMPTY + 1,
  V_FULL = P_FREE + 2,
  V_EMPTY = V_FULL + NVG,
  P_FULL = V_EMPTY + NVG,
  PV_TILE = P_FULL + 2,
  O_DONE = PV_TILE + 1,
  EVENT = O_DONE + 1,
  CORR_DONE = EVENT + 1,
  STATS = CORR_DONE + 1,
  DRAIN = STATS + 1,
  NBAR = DRAIN + 1
};
constexpr int OFF_TMEM = 512;           // u32 TMEM base
constexpr int OFF_ABORT = 516;          // u32 abort flag
constexpr int OFF_EVTYPE = 520;         // u32 event type (1 rescale, 2 done)     [PV]
constexpr int OFF_EVTILE = 524;         // u32 P slot of a rescale event           [PV]
constexpr int OFF_MFIN = 2048;          // f32 [128] final running max (log2)      [PV, remote]
constexpr int OFF_LFIN = 2560;          // f32 [128] final running sum             [PV, remote]
constexpr int OFF_XCH = 3072;           // f32 [2][128] max / sum exchange         [QK, local]
constexpr int OFF_ORDER = 1024;         // i32 [LPT_MAX] requests by length, at start only
constexpr int LPT_MAX = 256;            // longest-first dispatch for up to this many requests
static_assert(NBAR * 8 <= OFF_TMEM, "barrier block overflow");

constexpr int Q_OFF = CTRL;                           // Q chunk 8 (rope)
constexpr int STG_OFF = Q_OFF + (NCHUNK - NQT) * CHUNK; // P staging, 2 slots
constexpr int K_OFF = STG_OFF + 2 * PSLOT;
constexpr int QK_END = K_OFF + NK * KCHUNK;
constexpr int P_OFF = CTRL;
constexpr int V_OFF = P_OFF + 2 * PSLOT;
constexpr int PV_END = V_OFF + NVG * VG;
constexpr int PT_OFF = QK_END > PV_END ? QK_END : PV_END;   // paged caches: the unit's page slice
constexpr int PT_MAX = 2048;                                  // int32 entries (8 KB)
constexpr int SMEM_BYTES = PT_OFF + PT_MAX * 4 + 1024;
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

constexpr uint32_t IDESC_QK = idesc_bf16(BM, BQ, 0, 0);    // Q, K both K-major
constexpr uint32_t IDESC_PV = idesc_bf16(BM, 256, 0, 1);   // P K-major, V MN-major
constexpr float RESCALE_THRESHOLD = 8.0f;                  // log2 units: P <= 2^8
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;          // 2 s per wait

struct Params {
  const int32_t* cache_lens;
  const uint32_t* vis;
  const int32_t* positions;
  uint16_t* out;
  float* lse;
  float* part_o;
  float* part_lse;
  int32_t* err;
  int64_t cap;                    // logical slots per request (pages_per_req * P when paged)
  int B, n, H, W, mtiles, splits;
  float scale_log2;
  const int32_t* page_table;      // paged caches: [B][pages_per_req] physical page ids
  int page_size, page_shift, pages_per_req;   // page_size = 1 << page_shift
};

struct Ctx {
  uint32_t base;          // shared address of the aligned block
  volatile uint32_t* abort_flag;
  uint32_t peer;          // cluster rank of the other CTA
  int32_t* err;
  __device__ uint32_t bar(int i) const { return base + 8u * (uint32_t)i; }
};

__device__ __noinline__ void abort_pair(Ctx cx) {
  *cx.abort_flag = 1u;
  st_cluster_u32(map_to_rank(cx.base + OFF_ABORT, cx.peer), 1u);
  raise_dev_error(cx.err, KD_DEV_TIMEOUT);
}

// Bounded wait for the phase of `bar` with parity `par` to complete.
__device__ __forceinline__ bool wait_bar(const Ctx& cx, uint32_t bar, uint32_t par,
                                         bool cluster_scope = false) {
  if (cluster_scope ? mbar_try_wait_cluster(bar, par) : mbar_try_wait(bar, par)) return true;
  uint64_t t0 = 0;
  for (uint32_t spin = 1;; ++spin) {
    if (cluster_scope ? mbar_try_wait_cluster(bar, par) : mbar_try_wait(bar, par)) return true;
    if ((spin & 63u) == 0u) {
      if (*cx.abort_flag) return false;
      const uint64_t t = globaltimer();
      if (t0 == 0) t0 = t;
      else if (t - t0 > WAIT_LIMIT_NS) { abort_pair(cx); return false; }
    }
  }
}

// Warp-uniform outcome of a wait (all 32 lanes call it).
__device__ __forceinline__ bool wait_warp(const Ctx& cx, uint32_t bar, uint32_t par,
                                          bool cluster_scope = false) {
  return __all_sync(0xffffffffu, wait_bar(cx, bar, par, cluster_scope));
}

// Group-uniform outcome of a wait for the 256-thread group at named barrier 1.
__device__ __forceinline__ bool wait_group(const Ctx& cx, uint32_t bar, uint32_t par,
                                           bool cluster_scope = false) {
  const bool ok = wait_bar(cx, bar, par, cluster_scope);
  return !named_bar_red_or(1, GROUP, !ok);
}

// Shared-memory offset where TMA drops Q latent chunk c (0..7) at the start of a unit.
__host__ __device__ constexpr int q_stage_off(int c) {
  return c < 4 ? STG_OFF + c * CHUNK : K_OFF + 2 * KCHUNK + (c - 4) * CHUNK;
}
static_assert(4 * CHUNK <= 2 * PSLOT && 2 * KCHUNK + 4 * CHUNK <= NK * KCHUNK, "Q landing zones");

__device__ __forceinline__ uint64_t desc_k(uint32_t saddr) {      // K-major, SW128
  return smem_desc_sw128(saddr, 16, 1024);
}
__device__ __forceinline__ uint64_t desc_mn(uint32_t saddr) {     // MN-major, SW128, 8 KB atoms
  return smem_desc_sw128(saddr, VCH, 1024);
}

// Word q (0..3) of a node's visibility mask, without dynamic register indexing.
__device__ __forceinline__ uint32_t mask_word(const uint32_t (&w)[4], int q) {
  return q == 0 ? w[0] : (q == 1 ? w[1] : (q == 2 ? w[2] : w[3]));
}

__device__ __forceinline__ float max4(float a, float b, float c, float d) {
  return fmaxf(fmaxf(a, b), fmaxf(c, d));
}

// ====================================================================== QK CTA roles
// TMA producer: Q chunks 7 and 8 once, then the K ring.
// Cache row of request-relative key `key` of a paged cache (the unit's page-table
// slice is in shared memory from page page0 on; keys past the last page map to row
// 0: their scores are masked and their V rows never loaded).
__device__ __forceinline__ int32_t paged_row(const int32_t* ptab, int page0, const Params& p, int64_t key) {
  const int64_t pg = key >> p.page_shift;
  return pg < p.pages_per_req ? (ptab[pg - page0] << p.page_shift) + (int32_t)(key & (p.page_size - 1)) : 0;
}

template <bool PAGED>
__device__ __forceinline__ void qk_producer(const Ctx& cx, const Params& p, const int32_t* ptab,
                                            int page0, const CUtensorMap* tm_qa,
                                            const CUtensorMap* tm_qr, const CUtensorMap* tm_c,
                                            const CUtensorMap* tm_r, int qrow0, int64_t krow0,
                                            int64_t kbeg, int ntiles) {
  const uint32_t base = cx.base;
  // Q: latent chunks 0..3 land in the (still unused) P staging area, chunks 4..7 in
  // K ring stages 2..3; the softmax groups move them into TMEM.  The rope chunk stays.
  mbar_arrive_expect_tx(cx.bar(Q_FULL), NCHUNK * CHUNK);
  for (int c = 0; c < NQT; ++c) tma_load_2d(base + q_stage_off(c), tm_qa, c * KC, qrow0, cx.bar(Q_FULL));
  tma_load_2d(base + Q_OFF, tm_qr, 0, qrow0, cx.bar(Q_FULL));
  uint32_t it = 0;
  bool ok = true;
  for (int t = 0; t < ntiles && ok; ++t) {
    const int32_t krow = (int32_t)(krow0 + (int64_t)t * BQ);
    int32_t prow[4];                  // paged: the cache rows of the tile's (at most 4) pages
    if (PAGED) {
#pragma unroll
      for (int i = 0; i < 4; ++i)
        prow[i] = (i << p.page_shift) < BQ ? paged_row(ptab, page0, p, kbeg + (int64_t)t * BQ + (i << p.page_shift)) : 0;
    }
    for (int c = 0; c < NCHUNK; ++c, ++it) {
      const uint32_t st = it % NK, k = it / NK;
      if (!(ok = wait_bar(cx, cx.bar(K_EMPTY + st), (k & 1u) ^ 1u))) break;
      if (it == 2 && !(ok = wait_bar(cx, cx.bar(QT_FULL), 0))) break;   // stages 2, 3 held Q
      mbar_arrive_expect_tx(cx.bar(K_FULL + st), KCHUNK);
      const CUtensorMap* map = c < 8 ? tm_c : tm_r;
      const int x = c < 8 ? c * KC : 0;
      if (!PAGED) {
        tma_load_2d(base + K_OFF + st * KCHUNK, map, x, krow, cx.bar(K_FULL + st));
      } else {                        // one box per page (page_size rows, 1024-byte aligned)
#pragma unroll
        for (int i = 0; i < 4; ++i)
          if ((i << p.page_shift) < BQ)
            tma_load_2d(base + K_OFF + st * KCHUNK + (i << p.page_shift) * 128, map, x, prow[i],
                        cx.bar(K_FULL + st));
      }
    }
  }
  // every armed stage must have landed before the CTA may exit
  wait_bar(cx, cx.bar(Q_FULL), 0);
  for (uint32_t j = (it > NK ? it - NK : 0); j < it; ++j)
    wait_bar(cx, cx.bar(K_FULL + j % NK), (j / NK) & 1u);
}

// MMA issuer: S[t % 2] = Q K^T (A from TMEM for chunks 0..7, from shared memory for 8).
__device__ __forceinline__ void qk_mma(const Ctx& cx, uint32_t tmem, int ntiles) {
  const uint32_t base = cx.base;
  bool ok = wait_bar(cx, cx.bar(Q_FULL), 0) && wait_bar(cx, cx.bar(QT_FULL), 0);
  tc_fence_after();
  uint32_t it = 0;
  for (int t = 0; t < ntiles && ok; ++t) {
    if (!(ok = wait_bar(cx, cx.bar(S_EMPTY), (t & 1) ^ 1))) break;
    tc_fence_after();
    const uint32_t d = tmem + TS;
    for (int c = 0; c < NCHUNK; ++c, ++it) {
      const uint32_t st = it % NK;
      if (!(ok = wait_bar(cx, cx.bar(K_FULL + st), (it / NK) & 1u))) break;
      tc_fence_after();
      const uint32_t b0 = base + K_OFF + st * KCHUNK;
      if (c < NQT) {
#pragma unroll
        for (int kk = 0; kk < KC / 16; ++kk)
          mma_bf16_ts(d, tmem + TQ + c * 32 + kk * 8, desc_k(b0 + kk * 32), IDESC_QK, (c | kk) != 0);
      } else {
        const uint32_t a0 = base + Q_OFF + (c - NQT) * CHUNK;
#pragma unroll
        for (int kk = 0; kk < KC / 16; ++kk)
          mma_bf16_ss(d, desc_k(a0 + kk * 32), desc_k(b0 + kk * 32), IDESC_QK, 1u);
      }
      tc_commit(cx.bar(K_EMPTY + st));
    }
    if (ok) tc_commit(cx.bar(S_FULL));
  }
  tc_commit(cx.bar(DRAIN));
  wait_bar(cx, cx.bar(DRAIN), 0);
}

// One 128-key half of a QK tile: exponentiate this thread's 64 raw scores x as
// 2^(x s - mb) (s = softmax scale in log2 units, mb the scaled row reference),
// add them to the running sum, and ship the bf16 P tile (plus the per-row rescale
// factor for the PV side) through staging slot u % 2.
__device__ __forceinline__ bool emit_p(const Ctx& cx, uint8_t* gbase, const float (&x)[64], int u,
                                       float s, float mb, float alpha, bool rescale_row, int r, int g,
                                       uint32_t peer_p, uint32_t peer_ctrl, float& l_part) {
  const uint32_t sb = u & 1;
  float rs[4] = {0.f, 0.f, 0.f, 0.f};
  uint32_t pk[32];
  const float nmb = -mb;
#pragma unroll
  for (int c = 0; c < 32; ++c) {
    float a0, a1;
    ffma2(a0, a1, x[2 * c], x[2 * c + 1], s, nmb);
    const float p0 = ex2(a0), p1 = ex2(a1);
    fadd2(rs[2 * (c & 1)], rs[2 * (c & 1) + 1], p0, p1);
    pk[c] = pack_bf16x2(p0, p1);
  }
  l_part += (rs[0] + rs[1]) + (rs[2] + rs[3]);
  // staging slot sb (and the peer's P slot sb) is free once the PV MMAs of P tile u-2 completed
  if (!wait_group(cx, cx.bar(P_FREE + sb), ((u >> 1) & 1) ^ 1)) return false;
  const uint32_t stg = cx.base + STG_OFF + sb * PSLOT;
  const uint32_t prow = stg + g * (BM * 128) + (uint32_t)r * 128u;
#pragma unroll
  for (int q = 0; q < 8; ++q)
    st_shared_v4(prow + ((q ^ (r & 7)) << 4), pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
  float* stgf = reinterpret_cast<float*>(gbase + STG_OFF + sb * PSLOT);
  if (g == 0) stgf[(SLOT_ALPHA >> 2) + r] = alpha;
  fence_proxy_async_cta();
  const bool any = named_bar_red_or(1, GROUP, rescale_row);
  if (threadIdx.x == 64) {
    reinterpret_cast<uint32_t*>(stgf)[SLOT_FLAG >> 2] = any ? 1u : 0u;
    fence_proxy_async_cta();
    bulk_copy_to_peer(peer_p + sb * PSLOT, stg, SLOT_COPY, peer_ctrl + 8u * P_FULL + 8u * sb);
  }
  return true;
}

// Softmax groups: thread (g, r) owns row r and key columns [64 g, 64 g + 64) of every tile.
__device__ __forceinline__ void qk_softmax(const Ctx& cx, const Params& p, uint8_t* gbase,
                                           uint32_t tmem, int b, int mt, int sp, int64_t L,
                                           int64_t kbeg, int ntiles) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = (warp - 2) >> 2;
  const int quad = warp & 3;
  const int r = quad * 32 + lane;
  const uint32_t lane_addr = tmem + ((uint32_t)(quad * 32) << 16);
  const int n = p.n, H = p.H, rows_req = n * H;
  const int R = mt * BM + r;
  const bool valid = R < rows_req;
  const int node = valid ? R / H : 0;
  float* xch = reinterpret_cast<float*>(gbase + OFF_XCH);

  // ---- Q chunks 0..7 of this row into TMEM (group 0: chunks 0..3, group 1: 4..7),
  //      read back from the 128-byte-swizzled TMA landing zones
  {
    // an empty key partition issues no loads at all (its producer does not run)
    const bool okq = ntiles > 0 && wait_group(cx, cx.bar(Q_FULL), 0);
    if (okq) {
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) {
        const int c = g * 4 + c4;
        const uint8_t* row = gbase + q_stage_off(c) + r * 128;
        uint32_t v[32];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const uint4 x = *reinterpret_cast<const uint4*>(row + ((q ^ (r & 7)) << 4));
          v[4 * q] = x.x; v[4 * q + 1] = x.y; v[4 * q + 2] = x.z; v[4 * q + 3] = x.w;
        }
        tmem_st32(lane_addr + TQ + c * 32, v);
      }
      tmem_wait_st();
    }
    tc_fence_before();
    mbar_arrive(cx.bar(QT_FULL));
  }

  const int W = p.W;
  uint32_t w[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) w[q] = q < W ? p.vis[((size_t)b * n + node) * W + q] : 0u;
  if (g == 0 && valid && sp == 0 && (R % H) == 0) {
    const int depth = __popc(w[0]) + __popc(w[1]) + __popc(w[2]) + __popc(w[3]) - 1;
    if (!(w[0] & 1u) || !((mask_word(w, node >> 5) >> (node & 31)) & 1u)) raise_dev_error(p.err, KD_DEV_BAD_MASK);
    if (p.positions && p.positions[(size_t)b * n + node] != (int32_t)(L + depth))
      raise_dev_error(p.err, KD_DEV_BAD_POSITION);
  }
  const uint32_t peer_p = map_to_rank(cx.base + P_OFF, cx.peer);
  const uint32_t peer_ctrl = map_to_rank(cx.base, cx.peer);
  float m_ref = -INFINITY, l_part = 0.f;
  bool ok = true;
  for (int t = 0; t < ntiles && ok; ++t) {
    if (!(ok = wait_group(cx, cx.bar(S_FULL), t & 1))) break;
    tc_fence_after();
    // this thread's columns: keys 64 g .. 64 g + 63 of each 128-key half h of the tile
    float x[2][64];
    {
      uint32_t u0[64], u1[64];
      tmem_ld64(lane_addr + TS + g * 64, u0);
      tmem_ld64(lane_addr + TS + BN + g * 64, u1);
      tmem_wait_ld();
#pragma unroll
      for (int k = 0; k < 64; ++k) {            // raw scores: the scale is applied in emit_p
        x[0][k] = __uint_as_float(u0[k]);
        x[1][k] = __uint_as_float(u1[k]);
      }
    }
    tc_fence_before();
    mbar_arrive(cx.bar(S_EMPTY));              // TMEM free for the next tile's MMAs
    // mask: only keys at or beyond L need it
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int64_t kt = kbeg + (int64_t)t * BQ + h * BN + g * 64;
      if (kt + 64 > L) {
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const int64_t k = kt + c - L;
          bool vis_c = true;
          if (k >= 0) vis_c = (k < n) && ((mask_word(w, (int)k >> 5) >> ((int)k & 31)) & 1u);
          if (!vis_c) x[h][c] = -INFINITY;
        }
      }
    }
    // row max of the raw scores (the scale is positive, so it commutes with max)
    float mx[4] = {x[0][0], x[0][1], x[0][2], x[0][3]};
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int c = 0; c < 64; c += 8) {              // (re-reading x[0][0..3] is harmless)
        mx[0] = fmax3(mx[0], x[h][c], x[h][c + 4]);
        mx[1] = fmax3(mx[1], x[h][c + 1], x[h][c + 5]);
        mx[2] = fmax3(mx[2], x[h][c + 2], x[h][c + 6]);
        mx[3] = fmax3(mx[3], x[h][c + 3], x[h][c + 7]);
      }
    xch[g * BM + r] = max4(mx[0], mx[1], mx[2], mx[3]);
    named_bar_sync(1, GROUP);
    const float tmax = fmaxf(xch[r], xch[BM + r]) * p.scale_log2;
    float alpha = 1.f;
    bool rescale_row = false;
    if (tmax > m_ref + RESCALE_THRESHOLD) {
      if (m_ref != -INFINITY) {
        alpha = ex2(m_ref - tmax);
        rescale_row = true;
      } else {
        alpha = 0.f;
      }
      l_part *= alpha;
      m_ref = tmax;
    }
    const float mb = m_ref == -INFINITY ? 0.f : m_ref;
    ok = emit_p(cx, gbase, x[0], 2 * t, p.scale_log2, mb, alpha, rescale_row, r, g, peer_p, peer_ctrl,
                l_part) &&
         emit_p(cx, gbase, x[1], 2 * t + 1, p.scale_log2, mb, 1.f, false, r, g, peer_p, peer_ctrl, l_part);
  }
  // final row statistics for the epilogue: l = both groups' partial sums
  named_bar_sync(1, GROUP);
  xch[g * BM + r] = l_part;
  named_bar_sync(1, GROUP);
  if (g == 0) {
    st_cluster_u32(peer_ctrl + OFF_MFIN + r * 4, __float_as_uint(m_ref));
    st_cluster_u32(peer_ctrl + OFF_LFIN + r * 4, __float_as_uint(xch[r] + xch[BM + r]));
  }
  named_bar_sync(1, GROUP);
  if (threadIdx.x == 64) {
    mbar_arrive_remote(peer_ctrl + 8u * STATS);
    // the last P_FREE arrivals come from the peer's MMA completion: wait for them
    const int np = 2 * ntiles;
    if (ok)
      for (int u = (np > 2 ? np - 2 : 0); u < np; ++u)
        wait_bar(cx, cx.bar(P_FREE + (u & 1)), (u >> 1) & 1);
  }
}

// ====================================================================== PV CTA roles
// Keys of P tile t, key group kh that exist (the rest of the last QK tile lies past
// the request's last key).  Groups with none are neither loaded nor multiplied.
__device__ __forceinline__ int group_keys(int64_t kbeg, int64_t nkeys, int t, int kh) {
  const int64_t left = nkeys - (kbeg + (int64_t)t * BN + kh * VKEYS);
  return left <= 0 ? 0 : (left < VKEYS ? (int)left : VKEYS);
}

template <bool PAGED>
__device__ __forceinline__ void pv_producer(const Ctx& cx, const Params& p, const int32_t* ptab,
                                            int page0, const CUtensorMap* tm_v, int64_t krow0,
                                            int64_t kbeg, int64_t nkeys, int ntiles) {
  bool ok = true;
  uint32_t gi = 0;
  for (int t = 0; t < 2 * ntiles && ok; ++t) {
    for (int kh = 0; kh < BN / VKEYS && ok; ++kh) {
      if (group_keys(kbeg, nkeys, t, kh) == 0) continue;
      const int64_t key = kbeg + (int64_t)t * BN + kh * VKEYS;      // a 64-key group lies in one page
      const int32_t krow = PAGED ? paged_row(ptab, page0, p, key) : (int32_t)(krow0 + (key - kbeg));
      for (int hh = 0; hh < 2; ++hh, ++gi) {
        const uint32_t gs = gi % NVG, k = gi / NVG;
        if (!(ok = wait_bar(cx, cx.bar(V_EMPTY + gs), (k & 1u) ^ 1u))) break;
        mbar_arrive_expect_tx(cx.bar(V_FULL + gs), VG);
        for (int q = 0; q < 4; ++q)
          tma_load_2d(cx.base + V_OFF + gs * VG + q * VCH, tm_v, (hh * 4 + q) * KC, krow,
                      cx.bar(V_FULL + gs));
      }
    }
  }
  for (uint32_t j = (gi > NVG ? gi - NVG : 0); j < gi; ++j)
    wait_bar(cx, cx.bar(V_FULL + j % NVG), (j / NVG) & 1u);
}

__device__ __forceinline__ void pv_mma(const Ctx& cx, uint8_t* gbase, uint32_t tmem, int64_t kbeg,
                                       int64_t nkeys, int ntiles) {
  const int lane = threadIdx.x & 31;
  volatile uint32_t* ctrl = reinterpret_cast<volatile uint32_t*>(gbase);
  bool ok = true;
  uint32_t gi = 0, nres = 0;
  for (int t = 0; t < 2 * ntiles && ok; ++t) {      // P tiles of 128 keys
    const uint32_t sb = t & 1;
    if (lane == 0) mbar_arrive_expect_tx(cx.bar(P_FULL + sb), SLOT_COPY);
    if (!(ok = wait_warp(cx, cx.bar(P_FULL + sb), (t >> 1) & 1, true))) break;
    const uint32_t flag =
        *reinterpret_cast<volatile uint32_t*>(gbase + P_OFF + sb * PSLOT + SLOT_FLAG);
    if (flag && t > 0) {
      // every earlier PV MMA must be done before O is rescaled
      if (!(ok = wait_warp(cx, cx.bar(PV_TILE), (t - 1) & 1))) break;
      if (lane == 0) {
        ctrl[OFF_EVTYPE >> 2] = 1u;
        ctrl[OFF_EVTILE >> 2] = sb;
        mbar_arrive(cx.bar(EVENT));
      }
      if (!(ok = wait_warp(cx, cx.bar(CORR_DONE), nres & 1u))) break;
      ++nres;
    }
    tc_fence_after();
    for (int kh = 0; kh < BN / VKEYS && ok; ++kh) {
      const int nv = group_keys(kbeg, nkeys, t, kh);
      if (nv == 0) continue;             // P is zero there: nothing to add (and nothing loaded)
      for (int hh = 0; hh < 2 && ok; ++hh, ++gi) {
        const uint32_t gs = gi % NVG;
        if (!(ok = wait_warp(cx, cx.bar(V_FULL + gs), (gi / NVG) & 1u))) break;
        if (nv < VKEYS) {
          // rows past the request's last key may hold anything (even NaN bit
          // patterns); P is 0 there but 0 * NaN is not, so clear them.  A key row is
          // 128 contiguous bytes of its 64-column box (the swizzle stays inside a row).
          uint4* vg = reinterpret_cast<uint4*>(gbase + V_OFF + gs * VG);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            for (int e = nv * 8 + lane; e < VKEYS * 8; e += 32)
              vg[q * (VCH / 16) + e] = make_uint4(0u, 0u, 0u, 0u);
          fence_proxy_async_cta();
          __syncwarp();
        }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t pa = cx.base + P_OFF + sb * PSLOT + kh * (BM * 128);
          const uint32_t vb = cx.base + V_OFF + gs * VG;
#pragma unroll
          for (int ks = 0; ks < VKEYS / 16; ++ks)
            mma_bf16_ss(tmem + hh * 256, desc_k(pa + ks * 32), desc_mn(vb + ks * 2048), IDESC_PV,
                        (t > 0 || kh > 0 || ks > 0) ? 1u : 0u);
          tc_commit(cx.bar(V_EMPTY + gs));
        }
        __syncwarp();
      }
    }
    if (ok && lane == 0) {
      tc_commit(cx.bar(PV_TILE));
      tc_commit_mc(cx.bar(P_FREE + sb), (uint16_t)(1u << cx.peer));
    }
    __syncwarp();
  }
  if (lane == 0) {
    if (ntiles > 0) tc_commit(cx.bar(O_DONE));
    else mbar_arrive(cx.bar(O_DONE));
    ctrl[OFF_EVTYPE >> 2] = 2u;
    mbar_arrive(cx.bar(EVENT));
  }
  __syncwarp();
}

// Correction / epilogue groups: thread (g, r) owns row r, O columns [256 g, 256 g + 256).
__device__ __forceinline__ void pv_epilogue(const Ctx& cx, const Params& p, const CUtensorMap* tm_o,
                                            const CUtensorMap* tm_po, uint8_t* gbase, uint32_t tmem, int b, int mt, int sp,
                                            int ntiles) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = (warp - 2) >> 2;
  const int quad = warp & 3;
  const int r = quad * 32 + lane;
  const uint32_t lane_addr = tmem + ((uint32_t)(quad * 32) << 16) + g * 256;
  volatile uint32_t* ctrl = reinterpret_cast<volatile uint32_t*>(gbase);
  const volatile float* fctrl = reinterpret_cast<const volatile float*>(gbase);
  bool ok = true;
  uint32_t nev = 0;
  while (true) {
    if (!(ok = wait_group(cx, cx.bar(EVENT), nev & 1u))) break;
    ++nev;
    if (ctrl[OFF_EVTYPE >> 2] != 1u) break;
    const uint32_t sb = ctrl[OFF_EVTILE >> 2];
    const float a =
        reinterpret_cast<const volatile float*>(gbase + P_OFF + sb * PSLOT + SLOT_ALPHA)[r];
    tc_fence_after();
    uint32_t v[32];
    for (int c = 0; c < 256 / 32; ++c) {
      tmem_ld32(lane_addr + c * 32, v);
      tmem_wait_ld();
#pragma unroll
      for (int k = 0; k < 32; ++k) v[k] = __float_as_uint(__uint_as_float(v[k]) * a);
      tmem_st32(lane_addr + c * 32, v);
    }
    tmem_wait_st();
    tc_fence_before();
    mbar_arrive(cx.bar(CORR_DONE));
  }
  if (ok) ok = wait_group(cx, cx.bar(STATS), 0, true);
  if (ok) ok = wait_group(cx, cx.bar(O_DONE), 0);
  tc_fence_after();
  const float m = ok ? fctrl[(OFF_MFIN >> 2) + r] : 0.f;
  const float l = ok ? fctrl[(OFF_LFIN >> 2) + r] : 0.f;
  const int rows_req = p.n * p.H;
  const int R = mt * BM + r;
  const bool valid = ok && R < rows_req;
  const float inv = l > 0.f ? 1.f / l : 0.f;
  const bool have_o = ntiles > 0;
  const int64_t grow = (int64_t)b * rows_req + R;
  const int64_t prow = ((int64_t)sp * p.B * rows_req) + grow;     // row of part_lse
  if (p.splits == 1) {
    // bf16 tile -> eight 128-row x 64-column boxes in the (now idle) V ring, laid out
    // with the 128-byte swizzle, then TMA stores; the per-request 3-D tensor map
    // clips rows past the request's last node.
    for (int c = 0; c < 256 / 64; ++c) {
      uint32_t v[64];
      if (have_o && ok) {
        tmem_ld64(lane_addr + c * 64, v);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int k = 0; k < 64; ++k) v[k] = 0u;
      }
      const uint32_t box = cx.base + V_OFF + (g * 4 + c) * CHUNK + (uint32_t)r * 128u;
#pragma unroll
      for (int q = 0; q < 8; ++q)
        st_shared_v4(box + ((q ^ (r & 7)) << 4),
                     pack_bf16x2(__uint_as_float(v[8 * q + 0]) * inv, __uint_as_float(v[8 * q + 1]) * inv),
                     pack_bf16x2(__uint_as_float(v[8 * q + 2]) * inv, __uint_as_float(v[8 * q + 3]) * inv),
                     pack_bf16x2(__uint_as_float(v[8 * q + 4]) * inv, __uint_as_float(v[8 * q + 5]) * inv),
                     pack_bf16x2(__uint_as_float(v[8 * q + 6]) * inv, __uint_as_float(v[8 * q + 7]) * inv));
    }
    fence_proxy_async_cta();
    named_bar_sync(1, GROUP);
    if (threadIdx.x == 64 && ok) {
      for (int bx = 0; bx < 8; ++bx) tma_store_3d(tm_o, cx.base + V_OFF + bx * CHUNK, bx * KC, mt * BM, b);
      bulk_commit_group();
      bulk_wait_group_read0();
    }
  } else {
    // f32 partial tile in two rounds of eight 128-row x 32-column boxes (128-byte
    // swizzle) in the V ring; round k covers columns [256 g + 128 k, +128) of each
    // group.  The 3-D map [splits x B][rows][512] clips rows past the last node.
    for (int k = 0; k < 2; ++k) {
      if (k == 1) {
        if (threadIdx.x == 64 && ok) bulk_wait_group_read0();
        named_bar_sync(1, GROUP);
      }
      for (int h = 0; h < 2; ++h) {
        uint32_t v[64];
        if (have_o && ok) {
          tmem_ld64(lane_addr + k * 128 + h * 64, v);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int i = 0; i < 64; ++i) v[i] = 0u;
        }
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const uint32_t box = cx.base + V_OFF + (g * 4 + h * 2 + j) * CHUNK + (uint32_t)r * 128u;
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const int o = j * 32 + q * 4;
            st_shared_v4(box + ((q ^ (r & 7)) << 4), __float_as_uint(__uint_as_float(v[o]) * inv),
                         __float_as_uint(__uint_as_float(v[o + 1]) * inv),
                         __float_as_uint(__uint_as_float(v[o + 2]) * inv),
                         __float_as_uint(__uint_as_float(v[o + 3]) * inv));
          }
        }
      }
      fence_proxy_async_cta();
      named_bar_sync(1, GROUP);
      if (threadIdx.x == 64 && ok) {
        for (int bx = 0; bx < 8; ++bx)
          tma_store_3d(tm_po, cx.base + V_OFF + bx * CHUNK, (bx >> 2) * 256 + k * 128 + (bx & 3) * 32,
                       mt * BM, sp * p.B + b);
        bulk_commit_group();
        if (k == 1) bulk_wait_group_read0();
      }
    }
  }
  if (valid && g == 0) {
    const float lse_v = l > 0.f ? (m + __log2f(l)) * 0.69314718055994531f : -INFINITY;
    if (p.splits == 1) p.lse[grow] = lse_v;
    else p.part_lse[prow] = lse_v;
  }
  tc_fence_before();
}

// ====================================================================== kernel
template <bool PAGED>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NTHREADS, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tm_qa, const __grid_constant__ CUtensorMap tm_qr,
               const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_r,
               const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
               const __grid_constant__ CUtensorMap tm_po, const __grid_constant__ Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);

  const uint32_t rank = cluster_ctarank();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int unit = (int)cluster_id_x();
  const int mt = unit % p.mtiles;
  const int sp = (unit / p.mtiles) % p.splits;
  // Clusters are dispatched in index order; handing the longest requests out first
  // (their units stay adjacent, so their M tiles share K/V in L2) keeps the last
  // wave short when cache lengths differ.  Each CTA ranks the requests itself.
  int b = unit / (p.mtiles * p.splits);
  if (p.B > 1 && p.B <= LPT_MAX) {
    int* order = reinterpret_cast<int*>(gbase + OFF_ORDER);
    for (int i = threadIdx.x; i < p.B; i += blockDim.x) {
      const int li = p.cache_lens[i];
      int pos = 0;
      for (int j = 0; j < p.B; ++j) {
        const int lj = p.cache_lens[j];
        pos += (lj > li) || (lj == li && j < i);
      }
      order[pos] = i;
    }
    __syncthreads();
    b = order[b];
    __syncthreads();
  }
  const int n = p.n, H = p.H;

  const int64_t L = p.cache_lens[b];
  if (L < 0 || L + n > p.cap) {          // both CTAs see the same value and leave together
    if (rank == 0 && threadIdx.x == 0 && mt == 0 && sp == 0) raise_dev_error(p.err, KD_DEV_CACHE_FULL);
    return;
  }
  const int64_t nkeys = L + n;
  const int T = (int)((nkeys + BQ - 1) / BQ);         // 256-key QK tiles
  const int t0 = (int)((int64_t)sp * T / p.splits), t1 = (int)((int64_t)(sp + 1) * T / p.splits);
  const int ntiles = t1 - t0;
  const int64_t kbeg = (int64_t)t0 * BQ;                    // request-relative first key
  const int64_t krow0 = (int64_t)b * p.cap + kbeg;          // cache row of the first key
  const int qrow0 = b * n * H + mt * BM;

  Ctx cx;
  cx.base = base;
  cx.abort_flag = reinterpret_cast<volatile uint32_t*>(gbase + OFF_ABORT);
  cx.peer = rank ^ 1u;
  cx.err = p.err;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NBAR; ++i) {
      uint32_t cnt = 1;
      if (i == QT_FULL || i == S_EMPTY || i == CORR_DONE) cnt = GROUP;
      mbar_init(cx.bar(i), cnt);
    }
    *cx.abort_flag = 0u;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(base + OFF_TMEM, 512);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_qa);
    tma_prefetch_desc(&tm_qr);
    tma_prefetch_desc(&tm_c);
    tma_prefetch_desc(&tm_r);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_o);
    if (p.splits > 1) tma_prefetch_desc(&tm_po);
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(gbase + OFF_TMEM);

  // paged caches: the producer warp stages the page-table slice of this unit's keys
  const int32_t* ptab = reinterpret_cast<const int32_t*>(gbase + PT_OFF);
  const int page0 = PAGED ? (int)(kbeg / p.page_size) : 0;
  if (PAGED && warp == 0) {
    const int64_t kend = kbeg + (int64_t)ntiles * BQ;
    const int pend = (int)((kend + p.page_size - 1) / p.page_size);
    int32_t* dst = reinterpret_cast<int32_t*>(gbase + PT_OFF);
    for (int i = page0 + lane; i < pend && i < p.pages_per_req; i += 32)
      dst[i - page0] = p.page_table[(size_t)b * p.pages_per_req + i];
    __syncwarp();
  }

  if (rank == 0) {
    if (warp == 0) {
      if (lane == 0 && ntiles > 0)
        qk_producer<PAGED>(cx, p, ptab, page0, &tm_qa, &tm_qr, &tm_c, &tm_r, qrow0, krow0, kbeg, ntiles);
    } else if (warp == 1) {
      if (lane == 0 && ntiles > 0) qk_mma(cx, tmem, ntiles);
      __syncwarp();
    } else {
      qk_softmax(cx, p, gbase, tmem, b, mt, sp, L, kbeg, ntiles);
    }
  } else {
    if (warp == 0) {
      if (lane == 0) pv_producer<PAGED>(cx, p, ptab, page0, &tm_v, krow0, kbeg, nkeys, ntiles);
    } else if (warp == 1) {
      pv_mma(cx, gbase, tmem, kbeg, nkeys, ntiles);
    } else {
      pv_epilogue(cx, p, &tm_o, &tm_po, gbase, tmem, b, mt, sp, ntiles);
    }
  }

  // ------------------------------------------------------- teardown
  __syncwarp();          // the roles leave lanes behind (single-lane issuers, lane 64's waits)
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------ host side
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  }
  return fn;
}

// 2-D bf16 view [rows][inner] with `row_bytes` pitch, 64 x box_rows boxes, 128-byte swizzle.
static int make_map(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t rows, uint64_t row_bytes,
                    uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return KD_ELAUNCH;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {KC, box_rows};
  cuuint32_t es[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    set_cuda_error(cudaErrorInvalidValue, "cuTensorMapEncodeTiled");
    return KD_ELAUNCH;
  }
  return KD_OK;
}

// Per-request 3-D bf16 view [B][rows][512] of the output, 64 x 128 x 1 boxes, 128-byte swizzle.
static int make_out_map(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t B) {
  auto fn = encode_fn();
  if (!fn) return KD_ELAUNCH;
  cuuint64_t dims[3] = {KD_D_C, rows, B};
  cuuint64_t strides[2] = {KD_D_C * 2, rows * KD_D_C * 2};
  cuuint32_t box[3] = {KC, BM, 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    set_cuda_error(cudaErrorInvalidValue, "cuTensorMapEncodeTiled(out)");
    return KD_ELAUNCH;
  }
  return KD_OK;
}

// 3-D f32 view [splits x B][rows][512] of the split partials, 32 x 128 x 1 boxes,
// 128-byte swizzle.
static int make_part_map(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t zs) {
  auto fn = encode_fn();
  if (!fn) return KD_ELAUNCH;
  cuuint64_t dims[3] = {KD_D_C, rows, zs};
  cuuint64_t strides[2] = {KD_D_C * 4, rows * KD_D_C * 4};
  cuuint32_t box[3] = {32, BM, 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(ptr), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    set_cuda_error(cudaErrorInvalidValue, "cuTensorMapEncodeTiled(partial)");
    return KD_ELAUNCH;
  }
  return KD_OK;
}

// Co-resident 2-CTA clusters of the kernel on the current device (cached).
static int active_pairs(int sms) {
  static int cached[64];
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && cached[dev]) return cached[dev];
  int pairs = sms / 2;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  cfg.blockDim = dim3(NTHREADS, 1, 1);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cudaLaunchAttribute at;
  at.id = cudaLaunchAttributeClusterDimension;
  at.val.clusterDim.x = 2;
  at.val.clusterDim.y = 1;
  at.val.clusterDim.z = 1;
  cfg.attrs = &at;
  cfg.numAttrs = 1;
  int nc = 0;
  if (cudaOccupancyMaxActiveClusters(&nc, attn_tc_kernel<false>, &cfg) == cudaSuccess && nc > 0) pairs = nc;
  cudaGetLastError();
  if (dev >= 0 && dev < 64) cached[dev] = pairs;
  return pairs;
}

}  // namespace tc

// Split count for B requests of n nodes and H heads when the caller leaves it to
// the library: minimise waves x (tiles per unit + fixed cost) over the pairs that
// fit at once, with key length bounded by cap.
int auto_splits(int B, int n, int H, int64_t cap, int pairs) {
  const int64_t mtiles = ((int64_t)n * H + tc::BM - 1) / tc::BM;
  const int64_t units = (int64_t)B * mtiles;
  const int64_t T = (cap + tc::BQ - 1) / tc::BQ;
  int best = 1;
  double best_cost = 1e300;
  for (int s = 1; s <= 64 && s <= T; ++s) {
    const int64_t waves = (units * s + pairs - 1) / pairs;
    const double cost = (double)waves * ((double)((T + s - 1) / s) + 2.0) + (s > 1 ? 1.0 : 0.0);
    if (cost < best_cost * 0.98) { best_cost = cost; best = s; }
  }
  return best;
}

size_t workspace_bytes_for(int B, int n, int H, int splits) {
  size_t bytes = 256;
  if (splits > 1) {
    const size_t rows = (size_t)B * n * H;
    bytes += ((rows * splits * 4 + 255) / 256) * 256;       // partial lse
    bytes += rows * splits * KD_D_C * 4;                     // partial out
  }
  return bytes;
}

}  // namespace kd

using namespace kd;

extern "C" size_t kd_verify_workspace_bytes(int B, int n, int H, int64_t cap, int kv_splits) {
  if (!shapes_ok(B, n) || H < 1 || H > KD_MAX_HEADS || cap < 1 || kv_splits < 0 || kv_splits > 64) return 0;
  const int s = kv_splits > 0 ? kv_splits : auto_splits(B, n, H, cap, 74);
  return workspace_bytes_for(B, n, H, s);
}

// Both entry points: a contiguous cache (page_table == nullptr; cache rows B * cap) or a
// paged one (cache rows num_pages * page_size, cap = pages_per_req * page_size).
static int verify_attn_impl(const kd_bf16_t* q_abs, const kd_bf16_t* q_rope, const kd_bf16_t* c_kv,
                            const kd_bf16_t* k_rope, int64_t sc, int64_t sr, int64_t cap,
                            const int32_t* cache_lens, const uint32_t* vis, const int32_t* positions,
                            int B, int n, int H, float scale, kd_bf16_t* out, float* lse,
                            void* workspace, size_t ws_bytes, int kv_splits, const int32_t* page_table,
                            int page_size, int64_t pages_per_req, int64_t num_pages,
                            cudaStream_t stream) {
  const bool paged = page_table != nullptr;
  if (!q_abs || !q_rope || !cache_lens || !vis || !out || !lse || !workspace ||
      !shapes_ok(B, n) || H < 1 || H > KD_MAX_HEADS || !cache_ok(c_kv, k_rope, sc, sr, cap) ||
      !aligned16(q_abs) || !aligned16(q_rope) || !aligned16(out) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u) || !(scale > 0.f) || kv_splits < 0 ||
      kv_splits > 64)
    return KD_EINVAL;
  const int64_t rows = (int64_t)B * n * H;
  const int64_t cache_rows = paged ? num_pages * page_size : (int64_t)B * cap;
  if (rows > INT32_MAX || cache_rows > INT32_MAX) return KD_EINVAL;
  int sms = 0;
  int st = device_sms(&sms);
  if (st) return st;
  static bool attr_set[64];
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    st = cuda_status(cudaFuncSetAttribute(tc::attn_tc_kernel<false>,
                                          cudaFuncAttributeMaxDynamicSharedMemorySize, tc::SMEM_BYTES),
                     "cudaFuncSetAttribute(attn_tc_kernel)");
    if (st) return st;
    st = cuda_status(cudaFuncSetAttribute(tc::attn_tc_kernel<true>,
                                          cudaFuncAttributeMaxDynamicSharedMemorySize, tc::SMEM_BYTES),
                     "cudaFuncSetAttribute(attn_tc_kernel, paged)");
    if (st) return st;
    attr_set[dev] = true;
  }
  int splits = kv_splits;
  if (splits == 0) {
    splits = auto_splits(B, n, H, cap, tc::active_pairs(sms));
    while (splits > 1 && workspace_bytes_for(B, n, H, splits) > ws_bytes) --splits;
  }
  if (workspace_bytes_for(B, n, H, splits) > ws_bytes) return KD_ERANGE;

  CUtensorMap tq, tr, tcv, tkr, tv, to, tpo;
  if ((st = tc::make_map(&tq, q_abs, KD_D_C, (uint64_t)rows, KD_D_C * 2, tc::BM))) return st;
  if ((st = tc::make_map(&tr, q_rope, KD_D_R, (uint64_t)rows, KD_D_R * 2, tc::BM))) return st;
  const uint32_t kbox = paged ? (uint32_t)page_size : (uint32_t)tc::BQ;    // K box rows (one page)
  if ((st = tc::make_map(&tcv, c_kv, KD_D_C, (uint64_t)cache_rows, (uint64_t)sc * 2, kbox))) return st;
  if ((st = tc::make_map(&tkr, k_rope, KD_D_R, (uint64_t)cache_rows, (uint64_t)sr * 2, kbox))) return st;
  if ((st = tc::make_map(&tv, c_kv, KD_D_C, (uint64_t)cache_rows, (uint64_t)sc * 2, tc::VKEYS))) return st;
  if ((st = tc::make_out_map(&to, out, (uint64_t)rows / B, (uint64_t)B))) return st;

  tc::Params prm;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  prm.cache_lens = cache_lens;
  prm.vis = vis;
  prm.positions = positions;
  prm.out = out;
  prm.lse = lse;
  prm.err = reinterpret_cast<int32_t*>(ws);
  prm.part_lse = splits > 1 ? reinterpret_cast<float*>(ws + 256) : nullptr;
  prm.part_o = splits > 1 ? reinterpret_cast<float*>(ws + 256 + ((rows * splits * 4 + 255) / 256) * 256)
                          : nullptr;
  prm.cap = cap;
  prm.B = B;
  prm.n = n;
  prm.H = H;
  prm.W = (n + 31) / 32;
  prm.mtiles = (int)((rows / B + tc::BM - 1) / tc::BM);
  prm.splits = splits;
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.page_table = page_table;
  prm.page_size = paged ? page_size : 1;
  prm.page_shift = paged ? (page_size == 64 ? 6 : page_size == 128 ? 7 : 8) : 0;
  prm.pages_per_req = paged ? (int)pages_per_req : 0;
  if (splits > 1) {
    if ((st = tc::make_part_map(&tpo, prm.part_o, (uint64_t)rows / B, (uint64_t)splits * B))) return st;
  } else {
    tpo = to;                                   // not read with one split
  }
  const int64_t units = (int64_t)B * prm.mtiles * splits;
  if (2 * units > INT32_MAX) return KD_EINVAL;
  if (paged)
    tc::attn_tc_kernel<true><<<dim3((unsigned)(2 * units)), tc::NTHREADS, tc::SMEM_BYTES, stream>>>(
        tq, tr, tcv, tkr, tv, to, tpo, prm);
  else
    tc::attn_tc_kernel<false><<<dim3((unsigned)(2 * units)), tc::NTHREADS, tc::SMEM_BYTES, stream>>>(
        tq, tr, tcv, tkr, tv, to, tpo, prm);
  st = launch_status("attn_tc_kernel");
  if (st || splits == 1) return st;
  return launch_combine(prm.part_o, prm.part_lse, cache_lens, B, n, H, cap, splits, out, lse, stream);
}

extern "C" int kd_tree_verify_attn(const kd_bf16_t* q_abs, const kd_bf16_t* q_rope,
                                   const kd_bf16_t* c_kv, const kd_bf16_t* k_rope, int64_t sc,
                                   int64_t sr, int64_t cap, const int32_t* cache_lens,
                                   const uint32_t* vis, const int32_t* positions, int B, int n,
                                   int H, float scale, kd_bf16_t* out, float* lse, void* workspace,
                                   size_t ws_bytes, int kv_splits, cudaStream_t stream) {
  return verify_attn_impl(q_abs, q_rope, c_kv, k_rope, sc, sr, cap, cache_lens, vis, positions, B, n,
                          H, scale, out, lse, workspace, ws_bytes, kv_splits, nullptr, 1, 0, 0, stream);
}

extern "C" int kd_tree_verify_attn_paged(const kd_bf16_t* q_abs, const kd_bf16_t* q_rope,
                                         const kd_bf16_t* c_pages, const kd_bf16_t* r_pages,
                                         int64_t sc, int64_t sr, int page_size,
                                         const int32_t* page_table, int64_t pages_per_req,
                                         int64_t num_pages, const int32_t* cache_lens,
                                         const uint32_t* vis, const int32_t* positions, int B, int n,
                                         int H, float scale, kd_bf16_t* out, float* lse,
                                         void* workspace, size_t ws_bytes, int kv_splits,
                                         cudaStream_t stream) {
  if (!page_table || (page_size != 64 && page_size != 128 && page_size != 256) || pages_per_req < 1 ||
      pages_per_req + 1 > tc::PT_MAX || num_pages < 1)
    return KD_EINVAL;
  return verify_attn_impl(q_abs, q_rope, c_pages, r_pages, sc, sr, pages_per_req * page_size,
                          cache_lens, vis, positions, B, n, H, scale, out, lse, workspace, ws_bytes,
                          kv_splits, page_table, page_size, pages_per_req, num_pages, stream);
}

// ================================================================== allocation-free variant
// Some callers cannot allocate device memory when they verify: code running while
// a CUDA graph is being captured (allocation calls are not allowed there), serving
// loops that forbid allocator traffic on the hot path, and C hosts that embed this
// library without a device allocator of their own.  They use the entry point below,
// which takes its workspace from a fixed array that lives in this library instead
// of from the caller.  The array is KD_NOALLOC_SCRATCH_BYTES large and every GPU
// that loads the library keeps it until the process exits.
namespace kd {
static __device__ __align__(256) unsigned char g_noalloc_scratch[KD_NOALLOC_SCRATCH_BYTES];
}  // namespace kd

extern "C" int kd_tree_verify_attn_noalloc(const kd_bf16_t* q_nope_absorbed, const kd_bf16_t* q_rope,
                                           const kd_bf16_t* c_kv, const kd_bf16_t* k_rope,
                                           int64_t kv_row_stride_c, int64_t kv_row_stride_r,
                                           int64_t cap, const int32_t* cache_lens,
                                           const uint32_t* vis, const int32_t* positions, int B,
                                           int n, int H, float scale, kd_bf16_t* out, float* lse,
                                           int kv_splits, int32_t* dev_error, cudaStream_t stream) {
  // Requests that need more split-KV scratch than the array holds are refused here;
  // with kv_splits = 0 the automatic policy picks a split count that fits.
  if (kv_splits < 0 || kv_splits > 64) return KD_EINVAL;
  if (kv_splits > 0) {
    const size_t need = kd_verify_workspace_bytes(B, n, H, cap, kv_splits);
    if (need == 0) return KD_EINVAL;
    if (need > (size_t)KD_NOALLOC_SCRATCH_BYTES) return KD_ERANGE;
  }
  // Host code sees the array's name only as a stand-in, so the device address is
  // looked up once per device, with that device current, on the first call.
  static void* scratch_ptr[64];
  int dev = 0;
  int st = cuda_status(cudaGetDevice(&dev), "cudaGetDevice");
  if (st) return st;
  if (dev < 0 || dev >= 64) return KD_ENODEV;
  if (!scratch_ptr[dev]) {
    void* ptr = nullptr;
    st = cuda_status(cudaGetSymbolAddress(&ptr, kd::g_noalloc_scratch), "cudaGetSymbolAddress");
    if (st) return st;
    scratch_ptr[dev] = ptr;
  }
  void* scratch = scratch_ptr[dev];
  int32_t* err_word = static_cast<int32_t*>(scratch);   // first int32 of the workspace
  st = cuda_status(cudaMemsetAsync(err_word, 0, sizeof(int32_t), stream), "cudaMemsetAsync(error word)");
  if (st) return st;
  st = kd_tree_verify_attn(q_nope_absorbed, q_rope, c_kv, k_rope, kv_row_stride_c, kv_row_stride_r, cap,
                           cache_lens, vis, positions, B, n, H, scale, out, lse, scratch,
                           (size_t)KD_NOALLOC_SCRATCH_BYTES, kv_splits, stream);
  if (st) return st;
  if (dev_error)
    st = cuda_status(cudaMemcpyAsync(dev_error, err_word, sizeof(int32_t), cudaMemcpyDeviceToDevice, stream),
                     "cudaMemcpyAsync(error word)");
  return st;
}
