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
// 128-key P tiles.  A unit of work is (request, M tile, key partition).
//
// The fp32 output accumulator of one M tile (128 x 512) fills all 512 TMEM
// columns of an SM, leaving none for scores, so the kernel runs on 2-CTA clusters
// with split roles:
//   rank 0 ("QK" CTA): S = Q K^T for 256 keys at a time (M=128, N=256 MMAs) into
//       256 TMEM columns.  The eight 64-wide latent chunks of Q sit in the other 256
//       TMEM columns and feed the MMA as its A operand from tensor memory; the rope
//       chunk sits in shared memory.  A 4-stage ring of 32 KB stages carries K
//       (256 keys x 64 columns, TMA, 128-byte swizzle) and, at each unit boundary,
//       the next unit's Q latent (two 16 KB chunks per stage).  Two 4-warp softmax
//       groups copy S into registers (freeing TMEM for the next tile at once), take
//       the row max on raw scores, keep an online max with a lazy rescale
//       threshold, and emit P as two 128-key halves: each half is written into a
//       local staging slot in the K-major swizzled layout the MMA reads and moved
//       to rank 1 by a single bulk copy that completes on rank 1's barrier.  A tile
//       whose second half lies past the request's last key is computed by N=128
//       MMAs and sends only its first half.
//   rank 1 ("PV" CTA): O (128 x 512 fp32) in TMEM; V as 64-key x 256-column
//       groups (four 64-column MN-major boxes) in a 4-deep ring; O += P V as
//       M=128, N=256, K=16 MMAs; V groups wholly past the request's last key are
//       neither loaded nor multiplied.  Two 4-warp groups apply the rare O rescale
//       and write the normalised output (or a split's fp32 partial) as TMA box
//       stores staged through shared memory; a cluster's last unit stages through
//       the then idle P slots and V ring, many boxes in flight.
//
// The kernel is persistent: one cluster per SM pair.  Units are handed out
// dynamically from a global counter in longest-request-first order; each cluster's
// QK producer claims the next one while its current unit's last tile loads and
// publishes it to every role of both CTAs through a small ring in shared memory.
// Units overlap at their boundaries: the next unit's Q streams in behind the
// current unit's last K stages, and the output of one unit is written while the
// next one's scores are computed.  Key partitions of one M tile (split-KV, for
// short batches) are merged inside the same launch: each partition stores a
// normalised fp32 partial and bumps a per-tile ticket; after its last unit every
// CTA merges a fixed share of the rows once their tile's ticket is complete
// (log-sum-exp identity).
//
// attn_tc_kernel<true> reads a paged cache instead: each 256-key K stage arrives as
// one TMA box per page and each 64-key V group as one box inside a page, from the
// unit's slice of the page table staged in shared memory; page ids outside the
// pool are flagged (KD_DEV_BAD_PAGE) and that request's outputs are not written.
//
// Every wait is bounded (globaltimer); a wait that gives up raises KD_DEV_TIMEOUT,
// marks both CTAs aborted, and every role falls through to the common teardown
// (in-flight copies drained, cluster barrier, TMEM release).  No TMA multicast is
// used anywhere.

#include <cuda.h>
#include <cudaTypedefs.h>
#include <math.h>

#include <atomic>
#include <mutex>

#include "kd_common.cuh"
#include "kd_ptx.cuh"

namespace kd {
namespace tc {

using namespace ptx;

// ---------------------------------------------------------------- trace build
// Built with -DKD_TRACE (libkdverify_trace.so, "python -m
// tree_speculative_decoding_kd_b200.build --trace"), the kernel records, per CTA,
// the global timer at fixed points of each role (slots 0..31) and cycle counters
// of the main waits (slots 32..63); tree_speculative_decoding_kd_b200/trace.py names
// the slots and prints a launch's timeline.  The product library has none of it.
// Counters live in registers of the role's thread and reach memory once, when the
// role ends, so that they barely disturb what they measure.
#ifdef KD_TRACE
constexpr int TRACE_CTAS = 160, TRACE_SLOTS = 64;
__device__ unsigned long long g_trace[TRACE_CTAS][TRACE_SLOTS];
#define KD_EV(i) (g_trace[blockIdx.x][(i)] = globaltimer())
#define KD_CTR(c) long long c = 0
#define KD_T0(t) const long long t = clock64()
#define KD_ADD(c, t) ((c) += clock64() - (t))
#define KD_INC(c) (++(c))
#define KD_FLUSH(i, c) atomicAdd(&g_trace[blockIdx.x][(i)], (unsigned long long)(c))
#else
#define KD_EV(i) ((void)0)
#define KD_CTR(c) ((void)0)
#define KD_T0(t) ((void)0)
#define KD_ADD(c, t) ((void)0)
#define KD_INC(c) ((void)0)
#define KD_FLUSH(i, c) ((void)0)
#endif

constexpr int NTHREADS = 320;           // warp 0 TMA, warp 1 MMA, warps 2..9 two 4-warp groups
constexpr int GROUP = 256;              // threads of the two 4-warp groups
constexpr int BM = 128;                 // query rows per M tile
constexpr int BQ = 256;                 // keys per QK tile (S = 128 x 256)
constexpr int BN = 128;                 // keys per P / PV tile (two per QK tile)
constexpr int KC = 64;                  // columns per 128-byte swizzle atom
constexpr int NCHUNK = 9;               // 8 latent chunks + 1 rope chunk
constexpr int CHUNK = BN * KC * 2;      // 16 KB: 128 rows x 64 bf16
constexpr int KCHUNK = BQ * KC * 2;     // 32 KB: 256 keys x 64 bf16 (one ring stage)
constexpr int NQT = 8;                  // Q chunks held in TMEM (the rope chunk in shared memory)
constexpr int QSTAGES = NQT / 2;        // ring stages that carry a unit's Q latent
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
  K_FULL = 0,                           // QK: ring stage landed (TMA)
  K_EMPTY = K_FULL + NK,                // QK: ring stage consumed (MMA commit, or Q copied to TMEM)
  ROPE_FULL = K_EMPTY + NK,             // QK: the unit's Q rope chunk landed
  Q_FREE = ROPE_FULL + 1,               // QK: every MMA of a unit done (Q in TMEM and rope reusable)
  QT_FULL = Q_FREE + 1,                 // QK: the unit's Q latent is in TMEM (256 arrivals)
  S_FULL = QT_FULL + 1,                 // QK: S tile ready
  S_EMPTY = S_FULL + 1,                 // QK: S tile copied to registers (256 arrivals)
  P_FREE = S_EMPTY + 1,                 // QK: P slot sb consumed by the PV MMAs (2 slots)
  STATS_FREE = P_FREE + 2,              // QK: the PV side has read the last row statistics
  DRAIN = STATS_FREE + 1,               // QK: final MMA drain
  V_FULL = DRAIN + 1,                   // PV: V ring stage landed
  V_EMPTY = V_FULL + NVG,               // PV: V ring stage consumed
  P_FULL = V_EMPTY + NVG,               // PV: P slot sb arrived (bulk copy)
  STATS = P_FULL + 2,                   // PV: a unit's row statistics arrived
  O_DONE = STATS + 1,                   // PV: every PV MMA of a unit done
  O_FREE = O_DONE + 1,                  // PV: the epilogue has read O (256 arrivals)
  EVENT = O_FREE + 1,                   // PV: rescale or end-of-unit event for the epilogue
  CORR_DONE = EVENT + 1,                // PV: rescale applied (256 arrivals)
  PV_DRAIN = CORR_DONE + 1,             // PV: all issued PV MMAs done (before a rescale)
  SCHED_FULL = PV_DRAIN + 1,            // both: schedule slot k % NS published
  SCHED_EMPTY = SCHED_FULL + 4,         // QK: schedule slot read by all five consumers
  MERGE_FULL = SCHED_EMPTY + 4,         // both: a merge batch's partial rows landed (bulk copies)
  NBAR = MERGE_FULL + 1
};
constexpr int NS = 4;                   // schedule ring depth
constexpr int SCHED_READERS = 5;        // QK MMA, QK softmax, PV producer, PV MMA, PV epilogue
constexpr int OFF_TMEM = 512;           // u32 TMEM base
constexpr int OFF_ABORT = 516;          // u32 abort flag
constexpr int OFF_EVTYPE = 520;         // u32 event type (1 rescale, 2 end of unit)   [PV]
constexpr int OFF_EVTILE = 524;         // u32 P slot of a rescale event               [PV]
constexpr int OFF_SCHED = 544;          // i64 [NS] unit ranks of this cluster (-1: no more work)
constexpr int OFF_ORDER = 1024;         // i32 [LPT_MAX] requests by length
constexpr int OFF_MFIN = 2048;          // f32 [128] final running max (log2)          [PV, remote]
constexpr int OFF_LFIN = 2560;          // f32 [128] final running sum                 [PV, remote]
constexpr int OFF_XCH0 = 2048;          // f32 [2][128] max / sum exchange, even tiles [QK, local]
constexpr int OFF_XCH = 3072;           // f32 [2][128] max / sum exchange, odd tiles  [QK, local]
constexpr int LPT_MAX = 256;            // longest-first dispatch for up to this many requests
static_assert(NBAR * 8 <= OFF_TMEM, "barrier block overflow");

constexpr int Q_OFF = CTRL;                              // Q chunk 8 (rope)
constexpr int STG_OFF = Q_OFF + CHUNK;                   // P staging, 2 slots
constexpr int K_OFF = STG_OFF + 2 * PSLOT;
constexpr int QK_END = K_OFF + NK * KCHUNK;
constexpr int P_OFF = CTRL;
constexpr int V_OFF = P_OFF + 2 * PSLOT;
constexpr int EPI_OFF = V_OFF + NVG * VG;                 // epilogue staging, 2 KB per worker warp
constexpr int PV_END = EPI_OFF + 8 * 2048;
constexpr int EPI_RING = 12;                                  // last unit: 2 KB slots per warp in P + V
static_assert(8 * EPI_RING * 2048 <= EPI_OFF - P_OFF, "last-unit staging inside the P slots and V ring");
constexpr int PT_OFF = QK_END > PV_END ? QK_END : PV_END;   // paged caches: the unit's page slice
constexpr int PT_MAX = 2048;                                  // int32 entries (8 KB)
constexpr int SMEM_BYTES = PT_OFF + PT_MAX * 4 + 1024;
static_assert(SMEM_BYTES <= 232448, "shared memory budget");
static_assert(QSTAGES * KCHUNK == NQT * CHUNK && QSTAGES <= NK, "Q latent through the ring");

constexpr uint32_t IDESC_QK = idesc_bf16(BM, BQ, 0, 0);    // Q, K both K-major
constexpr uint32_t IDESC_QK_HALF = idesc_bf16(BM, BN, 0, 0); // a tile's first 128 keys only
constexpr uint32_t IDESC_PV = idesc_bf16(BM, 256, 0, 1);   // P K-major, V MN-major
constexpr float RESCALE_THRESHOLD = 8.0f;                  // log2 units: P <= 2^8
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;          // 2 s per wait

struct Params {
  const int32_t* cache_lens;
  const uint32_t* vis;
  const int32_t* positions;
  uint16_t* out;
  float* lse;
  float* part_o;                  // split partials [splits][B * n * H][512]
  float* part_lse;                // [splits][B * n * H]
  int32_t* tickets;               // [B * mtiles][2]: partitions stored, merges done
  int32_t* err;
  unsigned long long* sched;      // [0] ranks claimed after the first wave, [1] clusters done (self-resetting)
  int64_t cap;                    // logical slots per request (pages_per_req * P when paged)
  int64_t units;                  // B * mtiles * splits
  int B, n, H, W, mtiles, splits, clusters;
  float scale_log2;
  const int32_t* page_table;      // paged caches: [B][pages_per_req] physical page ids
  int page_size, page_shift, pages_per_req;   // page_size = 1 << page_shift
  int64_t num_pages;
};

struct Ctx {
  uint32_t base;          // shared address of the aligned block
  volatile uint32_t* abort_flag;
  uint32_t peer;          // cluster rank of the other CTA
  int32_t* err;
  __device__ uint32_t bar(int i) const { return base + 8u * (uint32_t)i; }
};

// Gives up on the pair: both CTAs' abort flags set, KD_DEV_TIMEOUT raised, and the
// wait that gave up recorded in the workspace's control block: the launch's first
// at byte 4, each warp's first at byte 32 + 4 (12 rank + warp); each word is bit 31
// set, CTA rank at bit 24, warp at bit 16, barrier index at bit 4, parity at bit 0
// (0 while nothing gave up).
__device__ __noinline__ void abort_pair(Ctx cx, uint32_t bar = 0u, uint32_t par = 0u) {
  *cx.abort_flag = 1u;
  st_cluster_u32(map_to_rank(cx.base + OFF_ABORT, cx.peer), 1u);
  raise_dev_error(cx.err, KD_DEV_TIMEOUT);
  const uint32_t rank = cluster_ctarank(), warp = threadIdx.x >> 5;
  const uint32_t site = 0x80000000u | (rank << 24) | (warp << 16) | (((bar - cx.base) >> 3) << 4) | (par & 1u);
  atomicCAS(reinterpret_cast<unsigned int*>(cx.err + 1), 0u, site);
  atomicCAS(reinterpret_cast<unsigned int*>(cx.err + 8 + 12 * rank + warp), 0u, site);
}

// Bounded wait for the phase of `bar` with parity `par` to complete.  With
// `drain`, the wait ignores the abort flag (used to let in-flight copies land
// before the CTA leaves) but keeps the time limit.
__device__ __forceinline__ bool wait_bar(const Ctx& cx, uint32_t bar, uint32_t par,
                                         bool cluster_scope = false, bool drain = false) {
  if (cluster_scope ? mbar_try_wait_cluster(bar, par) : mbar_try_wait(bar, par)) return true;
  uint64_t t0 = 0;
  for (uint32_t spin = 1;; ++spin) {
    if (cluster_scope ? mbar_try_wait_cluster(bar, par) : mbar_try_wait(bar, par)) return true;
    if ((spin & 63u) == 0u) {
      if (!drain && *cx.abort_flag) return false;
      const uint64_t t = globaltimer();
      if (t0 == 0) t0 = t;
      else if (t - t0 > WAIT_LIMIT_NS) {
        if (!drain) abort_pair(cx, bar, par);
        return false;
      }
    }
  }
}

// Warp-uniform outcome of a wait (all 32 lanes call it).
__device__ __forceinline__ bool wait_warp(const Ctx& cx, uint32_t bar, uint32_t par,
                                          bool cluster_scope = false) {
  return __all_sync(0xffffffffu, wait_bar(cx, bar, par, cluster_scope));
}

// Outcome of a wait made uniform over the 256 worker threads (named barrier 1);
// each thread may wait on its own barrier.
__device__ __forceinline__ bool wait_group(const Ctx& cx, uint32_t bar, uint32_t par,
                                           bool cluster_scope = false) {
  const bool ok = wait_bar(cx, bar, par, cluster_scope);
  return !named_bar_red_or(1, GROUP, !ok);
}

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

// Bits kt .. kt + 63 of the visibility string of one tree row, for the keys at
// and past the first tree slot L: key L + k is visible for k < 0 (committed
// keys), for 0 <= k < n when bit k of the row's mask (words m0..m3, zero past
// W) is set, and never for k >= n.
__device__ __noinline__ uint64_t vis_window(uint32_t m0, uint32_t m1, uint32_t m2, uint32_t m3, int n, int kt) {
  const uint32_t mw[4] = {m0, m1, m2, m3};
  uint32_t w[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int lo = 32 * q;
    const uint32_t keep = n >= lo + 32 ? ~0u : (n <= lo ? 0u : ((1u << (n - lo)) - 1u));
    w[q] = mw[q] & keep;
  }
  const uint64_t a = (uint64_t)w[0] | ((uint64_t)w[1] << 32), b = (uint64_t)w[2] | ((uint64_t)w[3] << 32);
  if (kt <= -64) return ~0ull;
  if (kt < 0) return (a << (-kt)) | ((1ull << (-kt)) - 1ull);
  if (kt == 0) return a;
  if (kt < 64) return (a >> kt) | (b << (64 - kt));
  if (kt < 128) return b >> (kt - 64);
  return 0ull;
}

__device__ __forceinline__ float max4(float a, float b, float c, float d) {
  return fmaxf(fmaxf(a, b), fmaxf(c, d));
}

// ====================================================================== units
struct Unit {
  int b, mt, sp, ntiles;
  int64_t L, kbeg, nkeys;
  bool valid;
};

// Unit of rank r: requests in `order` (longest first), then key partition, then M
// tile (the M tiles of one partition read the same keys and run side by side).
__device__ __forceinline__ Unit unit_at(const Params& p, const int* order, int64_t r) {
  Unit u;
  // 32-bit divisions (64-bit ones are long subroutines): ranks stay below 2^31 and
  // (sp + 1) * T below 64 * 2^23 since a key index fits 31 bits
  const int per_req = p.splits * p.mtiles;
  const int i = (int)r / per_req;
  const int loc = (int)r - i * per_req;
  u.sp = loc / p.mtiles;
  u.mt = loc - u.sp * p.mtiles;
  u.b = order ? order[i] : i;
  u.L = p.cache_lens[u.b];
  u.valid = u.L >= 0 && u.L + p.n <= p.cap;
  u.nkeys = u.L + p.n;
  const int T = u.valid ? (int)((u.nkeys + BQ - 1) / BQ) : 0;
  const int t0 = u.sp * T / p.splits, t1 = (u.sp + 1) * T / p.splits;
  u.ntiles = t1 - t0;
  u.kbeg = (int64_t)t0 * BQ;
  return u;
}

// ---------------------------------------------------------------- schedule ring
// Units are handed out dynamically: cluster c starts with rank c, then its QK
// producer claims ranks from a global counter (p.clusters onwards; longest requests
// first, see unit_at), skips those with no key tiles and
// publishes the k-th rank of its cluster in slot k % NS of a ring that both CTAs
// hold (the peer's copy written remotely); -1 ends the cluster's work.  Every role
// reads the ring in order and frees each slot once it has read it.
__device__ __forceinline__ volatile int64_t* sched_slots(uint8_t* gbase) {
  return reinterpret_cast<volatile int64_t*>(gbase + OFF_SCHED);
}

// Frees slot s from a role of this CTA (QK) or of the peer (PV).
__device__ __forceinline__ void sched_release(const Ctx& cx, int s, bool remote) {
  if (remote) mbar_arrive_remote(map_to_rank(cx.bar(SCHED_EMPTY + s), cx.peer));
  else mbar_arrive(cx.bar(SCHED_EMPTY + s));
}

// Rank the whole warp learns from lane 0's claims: the next rank with key tiles
// (requests whose cache does not fit raise KD_DEV_CACHE_FULL once), or -1.
__device__ __forceinline__ int64_t claim_unit(const Params& p, const int* order, int64_t first) {
  int64_t r = first;
  if ((threadIdx.x & 31) == 0) {
    while (r < p.units) {
      const Unit u = unit_at(p, order, r);
      if (u.ntiles > 0) break;
      if (!u.valid && u.mt == 0 && u.sp == 0) raise_dev_error(p.err, KD_DEV_CACHE_FULL);
      r = (int64_t)atomicAdd(p.sched, 1ull) + p.clusters;
    }
    if (r >= p.units) r = -1;
  }
  return __shfl_sync(0xffffffffu, r, 0);
}

// Cache row of request-relative key `key` of a paged cache (the unit's page-table
// slice is in shared memory from page page0 on; keys past the last page map to row
// 0: their scores are masked and their V rows never loaded).
__device__ __forceinline__ int32_t paged_row(const int32_t* ptab, int page0, const Params& p, int64_t key) {
  const int64_t pg = key >> p.page_shift;
  return pg < p.pages_per_req ? (ptab[pg - page0] << p.page_shift) + (int32_t)(key & (p.page_size - 1)) : 0;
}

// Pages [page0, pend) of request b staged into shared memory by one warp; ids
// outside the pool become page 0 (the request's outputs are not written: see
// request_pages_ok) so every TMA coordinate stays inside the pool.
__device__ __forceinline__ void stage_pages(const Params& p, int32_t* ptab, int b, int page0, int pend) {
  const int lane = threadIdx.x & 31;
  for (int i = page0 + lane; i < pend; i += 32) {
    const int32_t id = p.page_table[(size_t)b * p.pages_per_req + i];
    ptab[i - page0] = (id >= 0 && (int64_t)id < p.num_pages) ? id : 0;
  }
  __syncwarp();
}

// Whether every page id request b reads (pages [0, ceil(nkeys / P))) lies in the
// pool; all 256 worker threads call it.  A bad id sets KD_DEV_BAD_PAGE.
__device__ __forceinline__ bool request_pages_ok(const Params& p, int b, int64_t nkeys) {
  const int tid = threadIdx.x - 64;
  const int pend = (int)((nkeys + p.page_size - 1) >> p.page_shift);
  bool bad = false;
  for (int i = tid; i < pend && i < p.pages_per_req; i += GROUP) {
    const int32_t id = p.page_table[(size_t)b * p.pages_per_req + i];
    bad |= id < 0 || (int64_t)id >= p.num_pages;
  }
  bad = named_bar_red_or(1, GROUP, bad);
  if (bad && tid == 0) raise_dev_error(p.err, KD_DEV_BAD_PAGE);
  return !bad;
}

// ====================================================================== QK CTA roles
// TMA producer and scheduler (whole warp; lane 0 issues): claims the cluster's
// units and publishes them, then per unit loads the Q latent through four ring
// stages, the rope chunk of Q, and the K stages of every tile.
template <bool PAGED>
__device__ __forceinline__ void qk_producer(const Ctx& cx, const Params& p, const int* order, uint8_t* gbase,
                                            int32_t* ptab, const CUtensorMap* tm_qa,
                                            const CUtensorMap* tm_qr, const CUtensorMap* tm_c,
                                            const CUtensorMap* tm_r) {
  const int lane = threadIdx.x & 31;
  const uint32_t base = cx.base;
  volatile int64_t* slots = sched_slots(gbase);
  const uint32_t peer_slots = map_to_rank(base + OFF_SCHED, cx.peer);
  uint32_t it = 0, uq = 0;
  bool ok = true;
  // Q latent of unit u through four ring stages, then its rope chunk (whose buffer
  // is free once every MMA of the previous unit is done)
  auto load_q = [&](const Unit& u) -> bool {
    const int qrow0 = u.b * p.n * p.H + u.mt * BM;
    for (int q = 0; q < QSTAGES; ++q, ++it) {
      const uint32_t st = it % NK;
      if (!wait_warp(cx, cx.bar(K_EMPTY + st), ((it / NK) & 1u) ^ 1u)) return false;
      if (lane == 0) {
        mbar_arrive_expect_tx(cx.bar(K_FULL + st), KCHUNK);
        tma_load_2d(base + K_OFF + st * KCHUNK, tm_qa, 2 * q * KC, qrow0, cx.bar(K_FULL + st));
        tma_load_2d(base + K_OFF + st * KCHUNK + CHUNK, tm_qa, (2 * q + 1) * KC, qrow0, cx.bar(K_FULL + st));
      }
    }
    if (uq > 0 && !wait_warp(cx, cx.bar(Q_FREE), (uq - 1) & 1u)) return false;
    if (lane == 0) {
      mbar_arrive_expect_tx(cx.bar(ROPE_FULL), CHUNK);
      tma_load_2d(base + Q_OFF, tm_qr, 0, qrow0, cx.bar(ROPE_FULL));
    }
    ++uq;
    return true;
  };
  // cluster c starts with unit c (no claim on the way in); later units are claimed
  // from the counter, which hands out ranks from p.clusters on
  int64_t r = claim_unit(p, order, (int64_t)cluster_id_x());
  if (lane == 0) KD_EV(4);
  // the first unit's Q is requested before the unit is published: Q is the head of
  // the critical path, the other roles need the unit only later
  bool q_loaded = false;
  if (r >= 0) {
    if (!(ok = load_q(unit_at(p, order, r)))) r = -1;
    if (lane == 0) KD_EV(5);
    q_loaded = true;
  }
  for (int k = 0;; ++k) {
    // publish the k-th unit (or the end) once every role has read slot k - NS
    const int sl = k % NS;
    if (!(ok = wait_warp(cx, cx.bar(SCHED_EMPTY + sl), ((k / NS) & 1) ^ 1))) break;
    if (lane == 0) {
      slots[sl] = r;
      st_cluster_u32(peer_slots + sl * 8, (uint32_t)(uint64_t)r);
      st_cluster_u32(peer_slots + sl * 8 + 4, (uint32_t)((uint64_t)r >> 32));
      mbar_arrive(cx.bar(SCHED_FULL + sl));
      mbar_arrive_remote(map_to_rank(cx.bar(SCHED_FULL + sl), cx.peer));
    }
    if (lane == 0 && k == 0) KD_EV(6);
    __syncwarp();
    if (r < 0) break;
    const Unit u = unit_at(p, order, r);
    if (!q_loaded && !(ok = load_q(u))) break;
    q_loaded = false;
    const int page0 = PAGED ? (int)(u.kbeg >> p.page_shift) : 0;
    if (PAGED) {
      const int64_t kend = u.kbeg + (int64_t)u.ntiles * BQ;
      const int pend = (int)((kend + p.page_size - 1) >> p.page_shift);
      stage_pages(p, ptab, u.b, page0, pend < p.pages_per_req ? pend : p.pages_per_req);
    }
    const int64_t krow0 = (int64_t)u.b * p.cap + u.kbeg;
    int64_t claimed = 0;
    for (int t = 0; t < u.ntiles && ok; ++t) {
      const int32_t krow = (int32_t)(krow0 + (int64_t)t * BQ);
      int32_t prow[4];                // paged: the cache rows of the tile's (at most 4) pages
      if (PAGED) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
          prow[i] = (i << p.page_shift) < BQ
                        ? paged_row(ptab, page0, p, u.kbeg + (int64_t)t * BQ + (i << p.page_shift)) : 0;
      }
      // claim the next unit during the last tile, so the claim's latency is hidden
      if (t == u.ntiles - 1 && lane == 0) claimed = (int64_t)atomicAdd(p.sched, 1ull) + p.clusters;
      for (int c = 0; c < NCHUNK; ++c, ++it) {
        const uint32_t st = it % NK;
        if (!(ok = wait_warp(cx, cx.bar(K_EMPTY + st), ((it / NK) & 1u) ^ 1u))) break;
        if (lane == 0) {
          mbar_arrive_expect_tx(cx.bar(K_FULL + st), KCHUNK);
          const CUtensorMap* map = c < 8 ? tm_c : tm_r;
          const int x = c < 8 ? c * KC : 0;
          if (!PAGED) {
            tma_load_2d(base + K_OFF + st * KCHUNK, map, x, krow, cx.bar(K_FULL + st));
          } else {                    // one box per page (page_size rows, 1024-byte aligned)
#pragma unroll
            for (int i = 0; i < 4; ++i)
              if ((i << p.page_shift) < BQ)
                tma_load_2d(base + K_OFF + st * KCHUNK + (i << p.page_shift) * 128, map, x, prow[i],
                            cx.bar(K_FULL + st));
          }
        }
      }
    }
    if (!ok) break;
    if (lane == 0) KD_EV(7);
    r = claim_unit(p, order, claimed);
  }
  // every armed copy must land before the CTA may leave (bounded, even after an abort)
  if (lane == 0) {
    for (uint32_t j = (it > NK ? it - NK : 0); j < it; ++j)
      wait_bar(cx, cx.bar(K_FULL + j % NK), (j / NK) & 1u, false, true);
    if (uq > 0) wait_bar(cx, cx.bar(ROPE_FULL), (uq - 1) & 1u, false, true);
    // the last cluster to run out of work returns the counter to zero for the next launch
    if (atomicAdd(p.sched + 1, 1ull) == (unsigned long long)(p.clusters - 1)) {
      p.sched[0] = 0ull;
      p.sched[1] = 0ull;
    }
  }
  __syncwarp();
}

// MMA issuer: S = Q K^T per tile (A from TMEM for chunks 0..7, from shared memory
// for the rope chunk).
__device__ __forceinline__ void qk_mma(const Ctx& cx, const Params& p, const int* order, uint8_t* gbase,
                                       uint32_t tmem) {
  const uint32_t base = cx.base;
  volatile int64_t* slots = sched_slots(gbase);
  uint32_t it = 0, ts = 0, uq = 0;
  bool ok = true;
  KD_CTR(c_se);
  KD_CTR(c_kf);
  KD_CTR(c_is);
  KD_CTR(c_nt);
  KD_CTR(c_us);
  KD_CTR(c_qt);
  KD_CTR(c_nu);
  KD_CTR(c_f1);
  KD_CTR(c_sc);
  KD_CTR(c_tot);
  KD_T0(tall);
  KD_CTR(c_sw);
  KD_CTR(c_tile);
  KD_CTR(c_loop);
  for (int k = 0; ok; ++k) {
    KD_T0(tw);
    if (!(ok = wait_bar(cx, cx.bar(SCHED_FULL + k % NS), (k / NS) & 1, true))) break;
    const int64_t r = slots[k % NS];
    sched_release(cx, k % NS, false);
    if (k > 0) KD_ADD(c_sw, tw);
    if (r < 0) break;
    KD_T0(tu);
    const Unit u = unit_at(p, order, r);
    it += QSTAGES;                              // Q stages are consumed by the softmax groups
    KD_T0(tq);
    if (!(ok = wait_bar(cx, cx.bar(QT_FULL), uq & 1u) && wait_bar(cx, cx.bar(ROPE_FULL), uq & 1u))) break;
    KD_ADD(c_qt, tq);
    KD_ADD(c_us, tu);
    KD_INC(c_nu);
    if (uq == 0) KD_EV(8);
    tc_fence_after();
    KD_T0(tl);
    for (int t = 0; t < u.ntiles && ok; ++t, ++ts) {
      KD_T0(te);
      if (!(ok = wait_bar(cx, cx.bar(S_EMPTY), (ts & 1u) ^ 1u))) break;
      KD_ADD(c_se, te);
      KD_INC(c_nt);
      KD_T0(tf);
      tc_fence_after();
      const uint32_t d = tmem + TS;
      // a tile whose second half lies past the last key needs only its first 128 keys'
      // scores (the softmax masks the other columns, whatever they hold)
      const uint32_t idesc = u.kbeg + (int64_t)t * BQ + BN < u.nkeys ? IDESC_QK : IDESC_QK_HALF;
      for (int c = 0; c < NCHUNK; ++c, ++it) {
        const uint32_t st = it % NK;
        if (c == 0) KD_ADD(c_f1, tf);
        KD_T0(tk);
        if (!(ok = wait_bar(cx, cx.bar(K_FULL + st), (it / NK) & 1u))) break;
        KD_ADD(c_kf, tk);
        if (ts == 0 && c == 0) KD_EV(9);
        KD_T0(ti);
        tc_fence_after();
        const uint32_t b0 = base + K_OFF + st * KCHUNK;
        if (c < NQT) {
#pragma unroll
          for (int kk = 0; kk < KC / 16; ++kk)
            mma_bf16_ts(d, tmem + TQ + c * 32 + kk * 8, desc_k(b0 + kk * 32), idesc, (c | kk) != 0);
        } else {
#pragma unroll
          for (int kk = 0; kk < KC / 16; ++kk)
            mma_bf16_ss(d, desc_k(base + Q_OFF + kk * 32), desc_k(b0 + kk * 32), idesc, 1u);
        }
        tc_commit(cx.bar(K_EMPTY + st));
        KD_ADD(c_is, ti);
      }
      KD_T0(tc);
      if (ok) tc_commit(cx.bar(S_FULL));
      KD_ADD(c_sc, tc);
      KD_ADD(c_tile, te);
      if (ts == 0) KD_EV(10);
      KD_EV(11);
    }
    KD_ADD(c_loop, tl);
    if (ok) tc_commit(cx.bar(Q_FREE));
    ++uq;
  }
  KD_FLUSH(32, c_se);
  KD_FLUSH(33, c_kf);
  KD_FLUSH(34, c_is);
  KD_FLUSH(35, c_nt);
  KD_FLUSH(36, c_us);
  KD_FLUSH(37, c_qt);
  KD_FLUSH(38, c_nu);
  KD_FLUSH(47, c_f1);
  KD_FLUSH(48, c_sc);
  KD_FLUSH(50, c_sw);
  KD_FLUSH(51, c_tile);
  KD_FLUSH(52, c_loop);
  KD_ADD(c_tot, tall);
  KD_FLUSH(49, c_tot);
  tc_commit(cx.bar(DRAIN));
  wait_bar(cx, cx.bar(DRAIN), 0, false, true);
}

// Unit u's Q latent from its four ring stages (from ring position `pos`) into
// TMEM: group g moves chunks 4g..4g+3 of its row, then frees its two stages.
__device__ __forceinline__ bool copy_q(const Ctx& cx, uint8_t* gbase, uint32_t lane_addr, uint32_t pos,
                                       int g, int r) {
  bool ok = true;
#pragma unroll 1
  for (int s2 = 0; s2 < 2 && ok; ++s2) {
    const uint32_t s = pos + 2 * g + s2;
    if (!(ok = wait_group(cx, cx.bar(K_FULL + s % NK), (s / NK) & 1u))) break;
#pragma unroll 1
    for (int c2 = 0; c2 < 2; ++c2) {
      // in 8-column pieces: few registers, since the caller may hold a tile of scores
      const int chunk = 4 * g + 2 * s2 + c2;
      const uint8_t* row = gbase + K_OFF + (s % NK) * KCHUNK + c2 * CHUNK + r * 128;
#pragma unroll
      for (int q = 0; q < 8; q += 2) {
        const uint4 x = *reinterpret_cast<const uint4*>(row + ((q ^ (r & 7)) << 4));
        const uint4 y = *reinterpret_cast<const uint4*>(row + (((q + 1) ^ (r & 7)) << 4));
        tmem_st8(lane_addr + TQ + chunk * 32 + q * 4, x.x, x.y, x.z, x.w, y.x, y.y, y.z, y.w);
      }
    }
  }
  tmem_wait_st();
  named_bar_sync(1, GROUP);                     // every row of both groups read
  if (ok && (threadIdx.x & 127) == 0) {         // one thread per group frees its stages
    mbar_arrive(cx.bar(K_EMPTY + (pos + 2 * g) % NK));
    mbar_arrive(cx.bar(K_EMPTY + (pos + 2 * g + 1) % NK));
  }
  tc_fence_before();
  mbar_arrive(cx.bar(QT_FULL));
  return ok;
}

// One 128-key half of a QK tile: exponentiate this thread's 64 raw scores x as
// 2^(x s - mb) (s = softmax scale in log2 units, mb the scaled row reference),
// add them to the running sum, and ship the bf16 P tile (plus the per-row rescale
// factor for the PV side) through staging slot pc % 2.
__device__ __forceinline__ bool emit_p(const Ctx& cx, uint8_t* gbase, const float (&x)[64], uint32_t pc,
                                       float s, float mb, float alpha, bool rescale_row, int r, int g,
                                       uint32_t peer_p, uint32_t peer_ctrl, float& l_part) {
  const uint32_t sb = pc & 1;
  // staging slot sb (and the peer's P slot sb) is free once the PV MMAs of P tile pc-2 completed
  if (!wait_group(cx, cx.bar(P_FREE + sb), ((pc >> 1) & 1) ^ 1)) return false;
  const uint32_t stg = cx.base + STG_OFF + sb * PSLOT;
  const uint32_t prow = stg + g * (BM * 128) + (uint32_t)r * 128u;
  float rs[4] = {0.f, 0.f, 0.f, 0.f};
  const float nmb = -mb;
#pragma unroll
  for (int q = 0; q < 8; ++q) {             // 8 keys at a time, straight into the staging slot
    uint32_t pk[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int e = 8 * q + 2 * c;
      float a0, a1;
      ffma2(a0, a1, x[e], x[e + 1], s, nmb);
      const float p0 = ex2(a0), p1 = ex2(a1);
      fadd2(rs[2 * (c & 1)], rs[2 * (c & 1) + 1], p0, p1);
      pk[c] = pack_bf16x2(p0, p1);
    }
    st_shared_v4(prow + ((q ^ (r & 7)) << 4), pk[0], pk[1], pk[2], pk[3]);
  }
  l_part += (rs[0] + rs[1]) + (rs[2] + rs[3]);
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

// Softmax groups: thread (g, r) owns row r and key columns [64 g, 64 g + 64) of
// every 128-key half of every tile.
__device__ __forceinline__ bool qk_softmax(const Ctx& cx, const Params& p, const int* order, uint8_t* gbase,
                                           uint32_t tmem) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = (warp - 2) >> 2;
  const int quad = warp & 3;
  const int r = quad * 32 + lane;
  const uint32_t lane_addr = tmem + ((uint32_t)(quad * 32) << 16);
  const int n = p.n, H = p.H, rows_req = n * H, W = p.W;
  // two exchange buffers, alternating by tile, so a tile's writes never meet the
  // previous tile's reads
  const uint32_t xch0 = cx.base + OFF_XCH0;               // buffer b at xch0 + b * 1024
  const uint32_t peer_p = map_to_rank(cx.base + P_OFF, cx.peer);
  const uint32_t peer_ctrl = map_to_rank(cx.base, cx.peer);

  volatile int64_t* slots = sched_slots(gbase);
  uint32_t pos = 0, ts = 0, pc = 0, nq = 0, ns = 0;
  KD_CTR(c_sf);
  KD_CTR(c_em);
  KD_CTR(c_tt);
  bool ok = wait_group(cx, cx.bar(SCHED_FULL), 0, true);
  if (ok && slots[0] >= 0) ok = copy_q(cx, gbase, lane_addr, 0, g, r);     // the first unit's Q
  if (threadIdx.x == 64) KD_EV(12);
  for (int k = 0; ok; ++k) {
    if (!(ok = wait_group(cx, cx.bar(SCHED_FULL + k % NS), (k / NS) & 1, true))) break;
    const int64_t rk = slots[k % NS];
    named_bar_sync(1, GROUP);                   // every thread has read the slot
    if (threadIdx.x == 64) sched_release(cx, k % NS, false);
    if (rk < 0) break;
    const Unit u = unit_at(p, order, rk);
    float m_ref = -INFINITY, l_part = 0.f;
    {
      // this row's node (its mask is read again where a tile reaches the tree slots)
      const uint32_t* vrow;
      {
        const int R = u.mt * BM + r;
        const bool valid_row = R < rows_req;
        const int node = valid_row ? R / H : 0;
        vrow = p.vis + ((size_t)u.b * n + node) * W;
        if (g == 0 && valid_row && u.sp == 0 && (R % H) == 0) {
          uint32_t w[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) w[q] = q < W ? vrow[q] : 0u;
          const int depth = __popc(w[0]) + __popc(w[1]) + __popc(w[2]) + __popc(w[3]) - 1;
          if (!(w[0] & 1u) || !((mask_word(w, node >> 5) >> (node & 31)) & 1u))
            raise_dev_error(p.err, KD_DEV_BAD_MASK);
          if (p.positions && p.positions[(size_t)u.b * n + node] != (int32_t)(u.L + depth))
            raise_dev_error(p.err, KD_DEV_BAD_POSITION);
        }
      }
      const int rel0 = (int)(u.kbeg - u.L);     // first key of the unit relative to slot L
      for (int t = 0; t < u.ntiles && ok; ++t, ++ts) {
        // a tile reaching the tree slots needs the row's mask words: requested
        // before the wait for S so that their latency hides behind it
        uint32_t mw[4] = {0u, 0u, 0u, 0u};
        if (rel0 + (t + 1) * BQ > 0) {
#pragma unroll
          for (int q = 0; q < 4; ++q)
            if (q < W) mw[q] = vrow[q];
        }
        KD_T0(tsf);
        if (!(ok = wait_group(cx, cx.bar(S_FULL), ts & 1u))) break;
        KD_ADD(c_sf, tsf);
        if (threadIdx.x == 64) KD_EV(15);
        tc_fence_after();
        // this thread's columns: keys 64 g .. 64 g + 63 of each 128-key half h of the tile
        float x[2][64];
        {
          uint32_t u0[64], u1[64];
          tmem_ld64(lane_addr + TS + g * 64, u0);
          tmem_ld64(lane_addr + TS + BN + g * 64, u1);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 64; ++c) {         // raw scores: the scale is applied in emit_p
            x[0][c] = __uint_as_float(u0[c]);
            x[1][c] = __uint_as_float(u1[c]);
          }
        }
        tc_fence_before();
        mbar_arrive(cx.bar(S_EMPTY));            // TMEM free for the next tile's MMAs
        if (threadIdx.x == 64 && ts == 0) KD_EV(13);
        // mask: only keys at or beyond L need it.  The thread's 64 keys of half h
        // are one 64-bit window of the row's visibility bits; a clear bit sets the
        // score to -inf.  (Runs on one tile per unit, so it is kept compact: its
        // code is cold in the instruction cache every time it runs.)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          // key index relative to the first tree slot L (fits 32 bits: keys < 2^31)
          const int kt = rel0 + t * BQ + h * BN + g * 64;
          if (kt + 64 > 0) {
            const uint64_t vm = vis_window(mw[0], mw[1], mw[2], mw[3], n, kt);
            if (vm != ~0ull) {
              const uint32_t lo = (uint32_t)vm, hi = (uint32_t)(vm >> 32);
#pragma unroll
              for (int c = 0; c < 32; ++c) {
                if (!((lo >> c) & 1u)) x[h][c] = -INFINITY;
                if (!((hi >> c) & 1u)) x[h][c + 32] = -INFINITY;
              }
            }
          }
        }
        if (threadIdx.x == 64) KD_EV(16);
        // row max of the raw scores (the scale is positive, so it commutes with max)
        float mx[4] = {x[0][0], x[0][1], x[0][2], x[0][3]};
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int c = 0; c < 64; c += 8) {            // (re-reading x[0][0..3] is harmless)
            mx[0] = fmax3(mx[0], x[h][c], x[h][c + 4]);
            mx[1] = fmax3(mx[1], x[h][c + 1], x[h][c + 5]);
            mx[2] = fmax3(mx[2], x[h][c + 2], x[h][c + 6]);
            mx[3] = fmax3(mx[3], x[h][c + 3], x[h][c + 7]);
          }
        const uint32_t xch = xch0 + (ts & 1) * 1024;
        st_shared_f32(xch + (g * BM + r) * 4, max4(mx[0], mx[1], mx[2], mx[3]));
        named_bar_sync(1, GROUP);
        const float tmax = fmaxf(ld_shared_f32(xch + r * 4), ld_shared_f32(xch + (BM + r) * 4)) * p.scale_log2;
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
        KD_T0(tem);
        ok = emit_p(cx, gbase, x[0], pc, p.scale_log2, mb, alpha, rescale_row, r, g, peer_p, peer_ctrl,
                    l_part);
        if (ok && t == u.ntiles - 1) {
          // the last S of this unit is out of TMEM, so once its MMAs are done the next
          // unit's Q (if the schedule has one) may replace this one's; done with half
          // the scores already spent
          const int kn = k + 1;
          ok = wait_group(cx, cx.bar(SCHED_FULL + kn % NS), (kn / NS) & 1, true);
          if (ok && slots[kn % NS] >= 0)
            ok = wait_group(cx, cx.bar(Q_FREE), nq & 1u) &&
                 copy_q(cx, gbase, lane_addr, pos + QSTAGES + NCHUNK * (uint32_t)u.ntiles, g, r);
        }
        // the second half may lie wholly past the last key: then it is not sent
        if (u.kbeg + (int64_t)t * BQ + BN < u.nkeys) {
          ok = ok && emit_p(cx, gbase, x[1], pc + 1, p.scale_log2, mb, 1.f, false, r, g, peer_p, peer_ctrl,
                            l_part);
          pc += 2;
        } else {
          pc += 1;
        }
        KD_ADD(c_em, tem);
        KD_ADD(c_tt, tsf);
        if (threadIdx.x == 64) {
          if (ts == 0) KD_EV(14);
          KD_EV(17);
        }
      }
      if (!ok) break;
      pos += QSTAGES + NCHUNK * (uint32_t)u.ntiles;
      ++nq;
    }
    // final row statistics for the epilogue: l = both groups' partial sums (in the
    // exchange buffer the next tile will use)
    const uint32_t xch = xch0 + (ts & 1) * 1024;
    st_shared_f32(xch + (g * BM + r) * 4, l_part);
    named_bar_sync(1, GROUP);
    const float l_row = ld_shared_f32(xch + r * 4) + ld_shared_f32(xch + (BM + r) * 4);
    if (ns > 0 && !(ok = wait_group(cx, cx.bar(STATS_FREE), (ns - 1) & 1u))) break;
    if (g == 0) {
      st_cluster_u32(peer_ctrl + OFF_MFIN + r * 4, __float_as_uint(m_ref));
      st_cluster_u32(peer_ctrl + OFF_LFIN + r * 4, __float_as_uint(l_row));
    }
    named_bar_sync(1, GROUP);
    if (threadIdx.x == 64) mbar_arrive_remote(peer_ctrl + 8u * STATS);
    if (threadIdx.x == 64) KD_EV(18);
    ++ns;
  }
  if (threadIdx.x == 64) {
    KD_FLUSH(40, c_sf);
    KD_FLUSH(41, c_em);
    KD_FLUSH(42, c_tt);
  }
  // the peer's last arrivals on this CTA's barriers (P slots freed, statistics
  // read) must land before the CTA leaves
  if (threadIdx.x == 64) {
    for (uint32_t q = (pc > 2 ? pc - 2 : 0); q < pc; ++q)
      wait_bar(cx, cx.bar(P_FREE + (q & 1)), (q >> 1) & 1, false, true);
    if (ns > 0) wait_bar(cx, cx.bar(STATS_FREE), (ns - 1) & 1u, false, true);
  }
  return ok;
}

// ====================================================================== PV CTA roles
// Keys of P tile t, key group kh that exist (the rest of the last QK tile lies past
// the request's last key).  Groups with none are neither loaded nor multiplied.
__device__ __forceinline__ int group_keys(int64_t kbeg, int64_t nkeys, int t, int kh) {
  const int64_t left = nkeys - (kbeg + (int64_t)t * BN + kh * VKEYS);
  return left <= 0 ? 0 : (left < VKEYS ? (int)left : VKEYS);
}

template <bool PAGED>
__device__ __forceinline__ void pv_producer(const Ctx& cx, const Params& p, const int* order, uint8_t* gbase,
                                            int32_t* ptab, const CUtensorMap* tm_v) {
  const int lane = threadIdx.x & 31;
  volatile int64_t* slots = sched_slots(gbase);
  bool ok = true;
  uint32_t gi = 0;
  for (int k = 0; ok; ++k) {
    if (!(ok = wait_warp(cx, cx.bar(SCHED_FULL + k % NS), (k / NS) & 1, true))) break;
    const int64_t r = slots[k % NS];
    __syncwarp();
    if (lane == 0) sched_release(cx, k % NS, true);
    if (r < 0) break;
    const Unit u = unit_at(p, order, r);
    const int page0 = PAGED ? (int)(u.kbeg >> p.page_shift) : 0;
    if (PAGED) {
      const int64_t kend = u.kbeg + (int64_t)u.ntiles * BQ;
      const int pend = (int)((kend + p.page_size - 1) >> p.page_shift);
      stage_pages(p, ptab, u.b, page0, pend < p.pages_per_req ? pend : p.pages_per_req);
    }
    const int64_t krow0 = (int64_t)u.b * p.cap + u.kbeg;
    for (int t = 0; t < 2 * u.ntiles && ok; ++t) {
      for (int kh = 0; kh < BN / VKEYS && ok; ++kh) {
        if (group_keys(u.kbeg, u.nkeys, t, kh) == 0) continue;
        const int64_t key = u.kbeg + (int64_t)t * BN + kh * VKEYS;   // a 64-key group lies in one page
        const int32_t krow = PAGED ? paged_row(ptab, page0, p, key) : (int32_t)(krow0 + (key - u.kbeg));
        for (int hh = 0; hh < 2; ++hh, ++gi) {
          const uint32_t gs = gi % NVG;
          if (!(ok = wait_warp(cx, cx.bar(V_EMPTY + gs), ((gi / NVG) & 1u) ^ 1u))) break;
          if (lane == 0) {
            mbar_arrive_expect_tx(cx.bar(V_FULL + gs), VG);
            for (int q = 0; q < 4; ++q)
              tma_load_2d(cx.base + V_OFF + gs * VG + q * VCH, tm_v, (hh * 4 + q) * KC, krow,
                          cx.bar(V_FULL + gs));
            if (gi == 0) KD_EV(19);
          }
        }
      }
    }
  }
  if (lane == 0)
    for (uint32_t j = (gi > NVG ? gi - NVG : 0); j < gi; ++j)
      wait_bar(cx, cx.bar(V_FULL + j % NVG), (j / NVG) & 1u, false, true);
  __syncwarp();
}

__device__ __forceinline__ void pv_mma(const Ctx& cx, const Params& p, const int* order, uint8_t* gbase,
                                       uint32_t tmem) {
  const int lane = threadIdx.x & 31;
  volatile uint32_t* ctrl = reinterpret_cast<volatile uint32_t*>(gbase);
  volatile int64_t* slots = sched_slots(gbase);
  bool ok = true;
  uint32_t gi = 0, pc = 0, vu = 0, nres = 0, nd = 0;
  KD_CTR(c_pf);
  KD_CTR(c_vf);
  KD_CTR(c_nh);
  for (int k = 0; ok; ++k) {
    if (!(ok = wait_warp(cx, cx.bar(SCHED_FULL + k % NS), (k / NS) & 1, true))) break;
    const int64_t r = slots[k % NS];
    __syncwarp();
    if (lane == 0) sched_release(cx, k % NS, true);
    if (r < 0) break;
    const Unit u = unit_at(p, order, r);
    // the epilogue must have read the previous unit's O before it is overwritten
    if (vu > 0 && !(ok = wait_warp(cx, cx.bar(O_FREE), (vu - 1) & 1u))) break;
    for (int t = 0; t < 2 * u.ntiles && ok; ++t) {            // P tiles of 128 keys
      // a P tile wholly past the request's last key (the second half of a tile) is
      // neither sent by the QK CTA nor multiplied here; pc counts the tiles exchanged
      if (u.kbeg + (int64_t)t * BN >= u.nkeys) continue;
      const uint32_t sb = pc & 1;
      if (lane == 0) mbar_arrive_expect_tx(cx.bar(P_FULL + sb), SLOT_COPY);
      KD_T0(tp);
      if (!(ok = wait_warp(cx, cx.bar(P_FULL + sb), (pc >> 1) & 1, true))) break;
      KD_ADD(c_pf, tp);
      KD_INC(c_nh);
      if (lane == 0 && pc == 0) KD_EV(20);
      const uint32_t flag =
          *reinterpret_cast<volatile uint32_t*>(gbase + P_OFF + sb * PSLOT + SLOT_FLAG);
      if (flag && t > 0) {
        // every earlier PV MMA must be done before O is rescaled
        if (lane == 0) tc_commit(cx.bar(PV_DRAIN));
        if (!(ok = wait_warp(cx, cx.bar(PV_DRAIN), nd & 1u))) break;
        ++nd;
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
        const int nv = group_keys(u.kbeg, u.nkeys, t, kh);
        if (nv == 0) continue;             // P is zero there: nothing to add (and nothing loaded)
        for (int hh = 0; hh < 2 && ok; ++hh, ++gi) {
          const uint32_t gs = gi % NVG;
          KD_T0(tv);
          if (!(ok = wait_warp(cx, cx.bar(V_FULL + gs), (gi / NVG) & 1u))) break;
          KD_ADD(c_vf, tv);
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
      if (ok && lane == 0) tc_commit_mc(cx.bar(P_FREE + sb), (uint16_t)(1u << cx.peer));
      __syncwarp();
      ++pc;
    }
    if (!ok) break;
    if (lane == 0) {
      tc_commit(cx.bar(O_DONE));
      KD_EV(21);
      ctrl[OFF_EVTYPE >> 2] = 2u;
      mbar_arrive(cx.bar(EVENT));
    }
    __syncwarp();
    ++vu;
  }
  if (lane == 0) {
    KD_FLUSH(44, c_pf);
    KD_FLUSH(45, c_vf);
    KD_FLUSH(46, c_nh);
    tc_commit(cx.bar(PV_DRAIN));
    wait_bar(cx, cx.bar(PV_DRAIN), nd & 1u, false, true);
  }
  __syncwarp();
}

// Each lane holds 64 bytes (16 words) of its own row.  The warp writes its 32 rows
// into a 2 KB staging slot in the 64-byte swizzled layout of the output tensor map
// (16-byte piece c of row r at r * 64 + ((c ^ ((r >> 1) & 3)) << 4), which is also
// free of bank conflicts); a TMA store of the 32-row box then writes it out (rows
// past the request's last row are clipped by the map).
__device__ __forceinline__ void stage_row(uint32_t slot, const uint32_t (&w)[16]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int c = 0; c < 4; ++c)
    st_shared_v4(slot + lane * 64 + ((c ^ ((lane >> 1) & 3)) << 4), w[4 * c], w[4 * c + 1], w[4 * c + 2],
                 w[4 * c + 3]);
}

// One box through the warp's single slot, reused once the previous box has been
// read out of it.
__device__ __forceinline__ void warp_store_box(uint32_t stg, const uint32_t (&w)[16], const CUtensorMap* tm,
                                              int x, int y, int z, bool store) {
  const int lane = threadIdx.x & 31;
  if (lane == 0) bulk_wait_group_read0();
  __syncwarp();
  stage_row(stg, w);
  fence_proxy_async_cta();
  __syncwarp();
  if (lane == 0 && store) {
    tma_store_3d(tm, stg, x, y, z);
    bulk_commit_group();
  }
}

// Correction / epilogue groups: thread (g, r) owns row r, O columns [256 g, 256 g + 256).
__device__ __forceinline__ bool pv_epilogue(const Ctx& cx, const Params& p, const int* order, uint8_t* gbase,
                                            uint32_t tmem, bool paged, const CUtensorMap* tm_o) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = (warp - 2) >> 2;
  const int quad = warp & 3;
  const int r = quad * 32 + lane;
  const uint32_t lane_addr = tmem + ((uint32_t)(quad * 32) << 16) + g * 256;
  volatile uint32_t* ctrl = reinterpret_cast<volatile uint32_t*>(gbase);
  const volatile float* fctrl = reinterpret_cast<const volatile float*>(gbase);
  const uint32_t peer_ctrl = map_to_rank(cx.base, cx.peer);
  const int rows_req = p.n * p.H;
  volatile int64_t* slots = sched_slots(gbase);
  bool ok = true;
  uint32_t nev = 0, vu = 0;
  KD_CTR(c_es);
  KD_CTR(c_ew);
  KD_CTR(c_eu);
  for (int k = 0; ok; ++k) {
    if (!(ok = wait_group(cx, cx.bar(SCHED_FULL + k % NS), (k / NS) & 1, true))) break;
    const int64_t rk = slots[k % NS];
    named_bar_sync(1, GROUP);
    if (threadIdx.x == 64) sched_release(cx, k % NS, true);
    if (rk < 0) break;
    const Unit u = unit_at(p, order, rk);
    const bool pages_ok = !paged || request_pages_ok(p, u.b, u.nkeys);
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
        for (int q = 0; q < 32; ++q) v[q] = __float_as_uint(__uint_as_float(v[q]) * a);
        tmem_st32(lane_addr + c * 32, v);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(cx.bar(CORR_DONE));
    }
    if (!ok) break;
    if (!(ok = wait_group(cx, cx.bar(STATS), vu & 1u, true) && wait_group(cx, cx.bar(O_DONE), vu & 1u))) break;
    if (threadIdx.x == 64) KD_EV(22);
    // The cluster's next unit (or the end) is published once this unit's loads are
    // all issued, which O being complete implies, so this peek at the next schedule
    // slot cannot wait on anything the epilogue still has to do.  With no next unit
    // the P slots and the V ring are idle for good, and this unit's stores stage
    // through them (EPI_RING slots per warp, 64 columns per pass) instead of
    // through the warp's single 2 KB slot.
    const int kn = k + 1;
    if (!(ok = wait_group(cx, cx.bar(SCHED_FULL + kn % NS), (kn / NS) & 1, true))) break;
    const bool last = slots[kn % NS] < 0;
    tc_fence_after();
    const float m = fctrl[(OFF_MFIN >> 2) + r];
    const float l = fctrl[(OFF_LFIN >> 2) + r];
    named_bar_sync(1, GROUP);
    if (threadIdx.x == 64) mbar_arrive_remote(peer_ctrl + 8u * STATS_FREE);
    const int R = u.mt * BM + r;
    const bool write = pages_ok && R < rows_req;
    const float inv = l > 0.f ? 1.f / l : 0.f;
    const int64_t grow = (int64_t)u.b * rows_req + R;
    // this warp's 32 rows start at request row R0w of plane z of the output map
    // (request b, or partition sp of request b for split partials)
    const int R0w = u.mt * BM + quad * 32;
    const bool store = pages_ok && R0w < rows_req;
    const int z = p.splits == 1 ? u.b : u.sp * p.B + u.b;
    const uint32_t stg = last ? cx.base + P_OFF + (warp - 2) * (EPI_RING * 2048) : cx.base + EPI_OFF + (warp - 2) * 2048;
    KD_T0(tes);
    // Rolled loops over small TMEM reads: this code runs once per unit, so its size
    // (fetched cold every time) matters more than the exposed TMEM read latency.
    if (last) {
      // 64 columns per pass: two bf16 boxes or four fp32 boxes, one fence and one
      // commit group per pass; slots (pass * boxes + j) % EPI_RING
#pragma unroll 1
      for (int c = 0; c < 256 / 64; ++c) {
        uint32_t v[64];
        tmem_ld64(lane_addr + c * 64, v);
        tmem_wait_ld();
        if (c == 0 && threadIdx.x == 64) KD_EV(23);
        if (c == 256 / 64 - 1) {                // every TMEM read of this unit is done
          tc_fence_before();
          mbar_arrive(cx.bar(O_FREE));
        }
        // fp32 pass 3 reuses pass 0's slots: its boxes must be read out first
        if (lane == 0 && p.splits > 1 && c == 3) bulk_wait_group_read<2>();
        __syncwarp();
        if (p.splits == 1) {
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            uint32_t w[16];
#pragma unroll
            for (int q = 0; q < 16; ++q)
              w[q] = pack_bf16x2(__uint_as_float(v[32 * j + 2 * q]) * inv, __uint_as_float(v[32 * j + 2 * q + 1]) * inv);
            stage_row(stg + (2 * c + j) * 2048, w);
          }
        } else {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            uint32_t w[16];
#pragma unroll
            for (int q = 0; q < 16; ++q) w[q] = __float_as_uint(__uint_as_float(v[16 * j + q]) * inv);
            stage_row(stg + ((4 * c + j) % EPI_RING) * 2048, w);
          }
        }
        fence_proxy_async_cta();
        __syncwarp();
        if (lane == 0 && store) {
          if (p.splits == 1) {
            for (int j = 0; j < 2; ++j) tma_store_3d(tm_o, stg + (2 * c + j) * 2048, g * 256 + c * 64 + j * 32, R0w, z);
          } else {
            for (int j = 0; j < 4; ++j)
              tma_store_3d(tm_o, stg + ((4 * c + j) % EPI_RING) * 2048, g * 256 + c * 64 + j * 16, R0w, z);
          }
          bulk_commit_group();
        }
      }
    } else if (p.splits == 1) {                 // bf16: eight boxes of 32 columns
#pragma unroll 1
      for (int c = 0; c < 256 / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(lane_addr + c * 32, v);
        tmem_wait_ld();
        if (c == 256 / 32 - 1) {                // every TMEM read of this unit is done
          tc_fence_before();
          mbar_arrive(cx.bar(O_FREE));
        }
        uint32_t w[16];
#pragma unroll
        for (int q = 0; q < 16; ++q)
          w[q] = pack_bf16x2(__uint_as_float(v[2 * q]) * inv, __uint_as_float(v[2 * q + 1]) * inv);
        warp_store_box(stg, w, tm_o, g * 256 + c * 32, R0w, z, store);
      }
    } else {                                    // fp32: sixteen boxes of 16 columns
#pragma unroll 1
      for (int c = 0; c < 256 / 16; ++c) {
        uint32_t v[16];
        tmem_ld16(lane_addr + c * 16, v);
        tmem_wait_ld();
        if (c == 256 / 16 - 1) {
          tc_fence_before();
          mbar_arrive(cx.bar(O_FREE));
        }
        uint32_t w[16];
#pragma unroll
        for (int q = 0; q < 16; ++q) w[q] = __float_as_uint(__uint_as_float(v[q]) * inv);
        warp_store_box(stg, w, tm_o, g * 256 + c * 16, R0w, z, store);
      }
    }
    if (write && g == 0) {
      const float lse_v = l > 0.f ? (m + __log2f(l)) * 0.69314718055994531f : -INFINITY;
      if (p.splits == 1) p.lse[grow] = lse_v;
      else p.part_lse[(int64_t)u.sp * p.B * rows_req + grow] = lse_v;
    }
    if (p.splits > 1) {
      KD_ADD(c_es, tes);
      KD_T0(tew);
      // the partial is in global memory once every warp's boxes are written: publish
      // it on the tile's ticket
      if (lane == 0) {
        bulk_wait_group0();
        fence_proxy_async_global();
      }
      named_bar_sync(1, GROUP);
      if (threadIdx.x == 64) {
        __threadfence();
        atom_add_release_gpu(p.tickets + 2 * ((int64_t)u.b * p.mtiles + u.mt), 1);
      }
      KD_ADD(c_ew, tew);
      KD_INC(c_eu);
    }
    if (threadIdx.x == 64) KD_EV(24);
    ++vu;
  }
  if (lane == 0) bulk_wait_group0();            // every box stored before the CTA leaves
  __syncwarp();
  if (threadIdx.x == 64) {
    KD_FLUSH(58, c_es);
    KD_FLUSH(59, c_ew);
    KD_FLUSH(60, c_eu);
  }
  return ok;
}

// ====================================================================== split-KV merge
// Partition sp of request b covers QK tiles [sp T / S, (sp+1) T / S) of its T tiles;
// partitions without tiles are never scheduled and store nothing.
__device__ __forceinline__ bool partition_busy(int T, int sp, int S) {
  return (sp + 1) * T / S > sp * T / S;
}

// After its last unit, each CTA merges a fixed share of all rows (cluster c takes
// rows [c R / G, (c+1) R / G) of the R = B n H rows, split between its two CTAs),
// one M tile at a time once that tile's ticket shows every busy partition stored:
//   LSE = ln sum_s exp(lse_s),   out = sum_s exp(lse_s - LSE) o_s.
// The partial rows of a batch of rows are brought into shared memory by bulk copies
// all in flight at once (the P staging area and the K / V ring, idle by now: every
// load into them has landed and every MMA reading them is done), so a batch costs
// one memory round trip; each warp then merges rows from shared memory, lane l
// owning the 16-byte column pieces l, l + 32, l + 64, l + 96 of the 512-wide row.
// The merged-row count on the tile's second ticket word tells the last merger to
// return both words to zero for the next launch.
constexpr int MBUF_BYTES = 2 * PSLOT + NK * KCHUNK;        // STG + K ring (QK), P + V ring (PV)
constexpr int MBUF_ROWS = MBUF_BYTES / (KD_D_C * 4);       // partial rows the buffer holds
static_assert(2 * PSLOT + NVG * VG == MBUF_BYTES && STG_OFF + 2 * PSLOT == K_OFF && P_OFF + 2 * PSLOT == V_OFF,
              "merge buffer: one contiguous region in both CTAs");

__device__ __forceinline__ void merge_splits(const Ctx& cx, const Params& p, int cid, uint32_t rank,
                                             bool paged) {
  const int tid = threadIdx.x - 64;
  const int wid = tid >> 5, lane = threadIdx.x & 31;
  const int rows_req = p.n * p.H, S = p.splits;
  // 32-bit row arithmetic (B n H < 2^31): cluster c's share is q or q + 1 rows
  const int rows_all = p.B * rows_req;
  const int q_rows = rows_all / p.clusters, r_rows = rows_all - q_rows * p.clusters;
  const int lo = cid * q_rows + min(cid, r_rows), hi = lo + q_rows + (cid < r_rows ? 1 : 0);
  const int mid = (lo + hi) / 2;
  const int a = rank == 0 ? lo : mid, e = rank == 0 ? mid : hi;
  const uint32_t mbuf = cx.base + (rank == 0 ? STG_OFF : P_OFF);
  const int batch_rows = MBUF_ROWS / S;                      // S <= 64 < MBUF_ROWS
  uint32_t mph = 0;
  KD_CTR(c_mt);
  KD_CTR(c_ml);
  KD_CTR(c_mc);
  KD_CTR(c_mn);
  for (int row0 = a; row0 < e;) {
    const int b = row0 / rows_req;
    const int R0 = row0 - b * rows_req;
    const int mt = R0 / BM;
    const int rows_in = rows_req - mt * BM < BM ? rows_req - mt * BM : BM;
    const int tile_end_g = b * rows_req + mt * BM + rows_in;
    const int row1 = tile_end_g < e ? tile_end_g : e;
    const int64_t L = p.cache_lens[b];
    const bool valid = L >= 0 && L + p.n <= p.cap;
    if (valid) {
      const int64_t nkeys = L + p.n;
      const int T = (int)((nkeys + BQ - 1) / BQ);
      // busy partitions as a bit mask (lane l decides partitions l and l + 32)
      const bool s0 = lane < S && partition_busy(T, lane, S);
      const bool s1 = lane + 32 < S && partition_busy(T, lane + 32, S);
      const uint64_t busy_mask = (uint64_t)__ballot_sync(0xffffffffu, s0) |
                                 ((uint64_t)__ballot_sync(0xffffffffu, s1) << 32);
      const int busy = __popcll(busy_mask);
      int32_t* ticket = p.tickets + 2 * ((int64_t)b * p.mtiles + mt);
      // wait until every busy partition of the tile has stored its partial
      KD_T0(tmt);
      bool ok = true;
      if (tid == 0) {
        uint64_t t0 = 0;
        for (uint32_t spin = 1; ld_acquire_gpu(ticket) < busy; ++spin) {
          if ((spin & 63u) == 0u) {
            if (*cx.abort_flag) { ok = false; break; }
            const uint64_t t = globaltimer();
            if (t0 == 0) t0 = t;
            else if (t - t0 > WAIT_LIMIT_NS) { abort_pair(cx); ok = false; break; }
          }
        }
      }
      if (named_bar_red_or(1, GROUP, !ok)) return;
      KD_ADD(c_mt, tmt);
      KD_INC(c_mn);
#ifdef KD_TRACE
      if (threadIdx.x == 64 && g_trace[blockIdx.x][26] == 0) KD_EV(26);
#endif
      const bool pages_ok = !paged || request_pages_ok(p, b, nkeys);
      for (int bs = row0; bs < row1 && pages_ok; bs += batch_rows) {
        const int nb = row1 - bs < batch_rows ? row1 - bs : batch_rows;
        // slot (r, sp) of the buffer holds partial sp of row bs + r (busy partitions only)
        if (wid == 0) {
          if (lane == 0) mbar_arrive_expect_tx(cx.bar(MERGE_FULL), (uint32_t)(nb * busy) * (KD_D_C * 4));
          fence_proxy_async_global();             // the partials (acquired above) feed async copies
          __syncwarp();
          for (int i = lane; i < nb * S; i += 32) {
            const int r = i / S, sp = i - r * S;
            if ((busy_mask >> sp) & 1ull)
              bulk_load_global(mbuf + (uint32_t)i * (KD_D_C * 4),
                               p.part_o + ((int64_t)sp * rows_all + (bs + r)) * KD_D_C, KD_D_C * 4,
                               cx.bar(MERGE_FULL));
          }
        }
        // this warp's rows of the batch: the lse of its first two rows are requested
        // before the wait, so that their latency hides behind the copies'
        const int rw = wid;
        float l0 = -INFINITY, l1 = -INFINITY, l0n = -INFINITY, l1n = -INFINITY;
        if (rw < nb) {
          if (s0) l0 = __ldcg(p.part_lse + (int64_t)lane * rows_all + (bs + rw));
          if (s1) l1 = __ldcg(p.part_lse + (int64_t)(lane + 32) * rows_all + (bs + rw));
        }
        if (rw + GROUP / 32 < nb) {
          if (s0) l0n = __ldcg(p.part_lse + (int64_t)lane * rows_all + (bs + rw + GROUP / 32));
          if (s1) l1n = __ldcg(p.part_lse + (int64_t)(lane + 32) * rows_all + (bs + rw + GROUP / 32));
        }
        KD_T0(tml);
        const bool landed = wait_bar(cx, cx.bar(MERGE_FULL), mph & 1u, false, true);
        ++mph;
        if (named_bar_red_or(1, GROUP, !landed)) { abort_pair(cx); return; }
        KD_ADD(c_ml, tml);
        KD_T0(tmc);
        for (int r = rw; r < nb; r += GROUP / 32) {
          const int grow = bs + r;
          if (r == rw + GROUP / 32) {
            l0 = l0n;
            l1 = l1n;
          } else if (r != rw) {
            l0 = s0 ? __ldcg(p.part_lse + (int64_t)lane * rows_all + grow) : -INFINITY;
            l1 = s1 ? __ldcg(p.part_lse + (int64_t)(lane + 32) * rows_all + grow) : -INFINITY;
          }
          float mx = fmaxf(l0, l1);
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
          const float LOG2E = 1.4426950408889634f;
          const float w0 = mx == -INFINITY ? 0.f : ex2((l0 - mx) * LOG2E);
          const float w1 = mx == -INFINITY ? 0.f : ex2((l1 - mx) * LOG2E);
          float sum = w0 + w1;
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
          float acc[16];
#pragma unroll
          for (int q = 0; q < 16; ++q) acc[q] = 0.f;
          for (int sp = 0; sp < S; ++sp) {
            const float ws = __shfl_sync(0xffffffffu, sp < 32 ? w0 : w1, sp & 31);
            if (ws == 0.f) continue;              // empty or idle partition (uniform over the warp)
            const uint32_t src = mbuf + (uint32_t)(r * S + sp) * (KD_D_C * 4) + lane * 16;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const uint4 v = ld_shared_v4(src + q * 512);
              acc[4 * q + 0] = fmaf(ws, __uint_as_float(v.x), acc[4 * q + 0]);
              acc[4 * q + 1] = fmaf(ws, __uint_as_float(v.y), acc[4 * q + 1]);
              acc[4 * q + 2] = fmaf(ws, __uint_as_float(v.z), acc[4 * q + 2]);
              acc[4 * q + 3] = fmaf(ws, __uint_as_float(v.w), acc[4 * q + 3]);
            }
          }
          const float inv = sum > 0.f ? 1.f / sum : 0.f;
          uint16_t* dst = p.out + (int64_t)grow * KD_D_C + lane * 4;
#pragma unroll
          for (int q = 0; q < 4; ++q)
            st_global_v2(dst + q * 128, pack_bf16x2(acc[4 * q] * inv, acc[4 * q + 1] * inv),
                         pack_bf16x2(acc[4 * q + 2] * inv, acc[4 * q + 3] * inv));
          if (lane == 0) p.lse[grow] = sum > 0.f ? mx + __logf(sum) : -INFINITY;
        }
        named_bar_sync(1, GROUP);               // the buffer is read out before the next batch
        KD_ADD(c_mc, tmc);
      }
      const int mine = (int)(row1 - row0);
      if (tid == 0 && atomicAdd(ticket + 1, mine) + mine == rows_in) {
        ticket[0] = 0;
        ticket[1] = 0;
      }
    }
    row0 = row1;
  }
  if (threadIdx.x == 64) {
    KD_FLUSH(53, c_mt);
    KD_FLUSH(54, c_ml);
    KD_FLUSH(55, c_mc);
    KD_FLUSH(56, c_mn);
  }
}

// ====================================================================== kernel
template <bool PAGED>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NTHREADS, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tm_qa, const __grid_constant__ CUtensorMap tm_qr,
               const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_r,
               const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
               const __grid_constant__ Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);

  const uint32_t rank = cluster_ctarank();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cid = (int)cluster_id_x();
  if (threadIdx.x == 0) KD_EV(0);

  Ctx cx;
  cx.base = base;
  cx.abort_flag = reinterpret_cast<volatile uint32_t*>(gbase + OFF_ABORT);
  cx.peer = rank ^ 1u;
  cx.err = p.err;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NBAR; ++i) {
      uint32_t cnt = 1;
      if (i == QT_FULL || i == S_EMPTY || i == CORR_DONE || i == O_FREE) cnt = GROUP;
      if (i >= SCHED_EMPTY && i < SCHED_EMPTY + NS) cnt = SCHED_READERS;
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
  }
  // Longest request first: each CTA ranks the requests by cache length itself.
  const int* order = nullptr;
  if (p.B > 1 && p.B <= LPT_MAX) {
    int* ord = reinterpret_cast<int*>(gbase + OFF_ORDER);
    int* lens = reinterpret_cast<int*>(gbase + OFF_XCH);     // free until the roles start
    for (int i = threadIdx.x; i < p.B; i += blockDim.x) lens[i] = p.cache_lens[i];
    __syncthreads();
    for (int i = threadIdx.x; i < p.B; i += blockDim.x) {
      const int li = lens[i];
      int pos = 0;
      for (int j = 0; j < p.B; ++j) {
        const int lj = lens[j];
        pos += (lj > li) || (lj == li && j < i);
      }
      ord[pos] = i;
    }
    order = ord;
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(gbase + OFF_TMEM);
  int32_t* ptab = reinterpret_cast<int32_t*>(gbase + PT_OFF);
  if (threadIdx.x == 0) KD_EV(1);

  bool ok = true;
  if (rank == 0) {
    if (warp == 0) {
      qk_producer<PAGED>(cx, p, order, gbase, ptab, &tm_qa, &tm_qr, &tm_c, &tm_r);
    } else if (warp == 1) {
      if (lane == 0) qk_mma(cx, p, order, gbase, tmem);
      __syncwarp();
    } else {
      ok = qk_softmax(cx, p, order, gbase, tmem);
    }
  } else {
    if (warp == 0) {
      pv_producer<PAGED>(cx, p, order, gbase, ptab, &tm_v);
    } else if (warp == 1) {
      pv_mma(cx, p, order, gbase, tmem);
    } else {
      ok = pv_epilogue(cx, p, order, gbase, tmem, PAGED, &tm_o);
    }
  }
  if (threadIdx.x == 64) KD_EV(25);
  if (warp >= 2 && p.splits > 1 && !named_bar_red_or(1, GROUP, !ok || *cx.abort_flag))
    merge_splits(cx, p, cid, rank, PAGED);
  if (threadIdx.x == 64) KD_EV(27);

  // ------------------------------------------------------- teardown
  __syncwarp();          // the roles leave lanes behind (single-lane issuers, lane 64's waits)
  __syncthreads();
  cluster_sync();
  if (threadIdx.x == 0) KD_EV(2);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
    if (lane == 0) KD_EV(3);
  }
}

// ------------------------------------------------------------------ host side
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

// Output map [planes][rows_req][512] (bf16 outputs, or fp32 split partials) stored in
// 32-row boxes of 64 bytes per row, 64-byte swizzle.
static int make_out_map(CUtensorMap* m, void* ptr, bool fp32, uint64_t rows_req, uint64_t planes) {
  auto fn = encode_fn();
  if (!fn) return KD_ELAUNCH;
  const uint64_t es = fp32 ? 4 : 2;
  cuuint64_t dims[3] = {KD_D_C, rows_req, planes};
  cuuint64_t strides[2] = {KD_D_C * es, rows_req * KD_D_C * es};
  cuuint32_t box[3] = {(cuuint32_t)(64 / es), 32, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, fp32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, ptr, dims,
                  strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                  CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    set_cuda_error(cudaErrorInvalidValue, "cuTensorMapEncodeTiled(out)");
    return KD_ELAUNCH;
  }
  return KD_OK;
}

// Co-resident 2-CTA clusters of the kernel on the current device (cached per device).
static int active_pairs(int sms) {
  static std::atomic<int> cached[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return sms / 2;
  }
  const int c = cached[dev].load(std::memory_order_relaxed);
  if (c > 0) return c;
  int pairs = sms / 2;
  if (cudaFuncSetAttribute(attn_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           SMEM_BYTES) == cudaSuccess) {
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
  }
  cudaGetLastError();
  cached[dev].store(pairs, std::memory_order_relaxed);
  return pairs;
}

}  // namespace tc

// Split count for B requests of n nodes and H heads when the caller leaves it to
// the library.  The persistent kernel runs `pairs` clusters; with S partitions per
// request there are B * mtiles * S units of about T / S tiles each, plus a fixed
// cost per unit (its boundary) and, when S > 1, the partial store and merge.  The
// split count minimising waves x (tiles per unit + fixed costs) wins, with key
// length bounded by cap.
int auto_splits(int B, int n, int H, int64_t cap, int pairs) {
  const int64_t mtiles = ((int64_t)n * H + tc::BM - 1) / tc::BM;
  const int64_t units = (int64_t)B * mtiles;
  const int64_t T = (cap + tc::BQ - 1) / tc::BQ;
  int best = 1;
  double best_cost = 1e300;
  for (int s = 1; s <= 64 && s <= T; ++s) {
    const int64_t waves = (units * s + pairs - 1) / pairs;
    const double cost = (double)waves * ((double)((T + s - 1) / s) + 0.5 + (s > 1 ? 1.0 : 0.0));
    if (cost < best_cost * 0.98) { best_cost = cost; best = s; }
  }
  return best;
}

// Workspace: 256-byte control block (int32 error word at byte 0, the first wait
// that gave up at byte 4, each warp's at bytes 32..127; the unit counter and the
// count of clusters out of work, two uint64 at bytes 8 and 16,
// which every launch returns to zero), then, with splits:
// per-M-tile tickets [B * mtiles][2] int32, partial lse [S][rows] and partial
// outputs [S][rows][512] fp32.
struct WsLayout {
  size_t tickets, part_lse, part_o, total;
};
static WsLayout ws_layout(int B, int n, int H, int splits) {
  WsLayout w;
  const size_t rows = (size_t)B * n * H;
  const size_t mtiles = ((size_t)n * H + tc::BM - 1) / tc::BM;
  w.tickets = 256;
  w.part_lse = w.tickets + ((B * mtiles * 8 + 255) / 256) * 256;
  w.part_o = w.part_lse + ((rows * splits * 4 + 255) / 256) * 256;
  w.total = splits > 1 ? w.part_o + rows * splits * KD_D_C * 4 : 256;
  return w;
}

size_t workspace_bytes_for(int B, int n, int H, int splits) { return ws_layout(B, n, H, splits).total; }

// Split count the call picks for kv_splits = 0 on the current device (74 pairs
// when no device is usable, e.g. on a build host).
int default_splits(int B, int n, int H, int64_t cap) {
  int sms = 0;
  const int pairs = device_sms(&sms) == KD_OK ? tc::active_pairs(sms) : 74;
  cudaGetLastError();
  return auto_splits(B, n, H, cap, pairs);
}

}  // namespace kd

using namespace kd;

#ifdef KD_TRACE
// Trace build only: copy out / clear the per-CTA trace of the last launches.
extern "C" int kd_trace_read(unsigned long long* host, size_t bytes) {
  if (bytes > sizeof(tc::g_trace)) bytes = sizeof(tc::g_trace);
  return cuda_status(cudaMemcpyFromSymbol(host, tc::g_trace, bytes), "cudaMemcpyFromSymbol(trace)");
}
extern "C" int kd_trace_clear(cudaStream_t stream) {
  void* ptr = nullptr;
  int st = cuda_status(cudaGetSymbolAddress(&ptr, tc::g_trace), "cudaGetSymbolAddress(trace)");
  if (st) return st;
  return cuda_status(cudaMemsetAsync(ptr, 0, sizeof(tc::g_trace), stream), "cudaMemsetAsync(trace)");
}
extern "C" int kd_trace_dims(int* ctas, int* slots) {
  *ctas = tc::TRACE_CTAS;
  *slots = tc::TRACE_SLOTS;
  return KD_OK;
}
#endif

extern "C" size_t kd_verify_workspace_bytes(int B, int n, int H, int64_t cap, int kv_splits) {
  if (!shapes_ok(B, n) || H < 1 || H > KD_MAX_HEADS || cap < 1 || kv_splits < 0 || kv_splits > 64) return 0;
  const int s = kv_splits > 0 ? kv_splits : default_splits(B, n, H, cap);
  return workspace_bytes_for(B, n, H, s);
}

// Argument checks shared by the entry points (nothing is enqueued).
static int check_attn_args(const kd_bf16_t* q_abs, const kd_bf16_t* q_rope, const kd_bf16_t* c_kv,
                           const kd_bf16_t* k_rope, int64_t sc, int64_t sr, int64_t cap,
                           const int32_t* cache_lens, const uint32_t* vis, int B, int n, int H, float scale,
                           const kd_bf16_t* out, const float* lse, int kv_splits, int64_t cache_rows) {
  if (!q_abs || !q_rope || !cache_lens || !vis || !out || !lse || !shapes_ok(B, n) || H < 1 ||
      H > KD_MAX_HEADS || !cache_ok(c_kv, k_rope, sc, sr, cap) || !aligned16(q_abs) || !aligned16(q_rope) ||
      !aligned16(out) || !(scale > 0.f) || kv_splits < 0 || kv_splits > 64)
    return KD_EINVAL;
  const int64_t rows = (int64_t)B * n * H;
  if (rows > INT32_MAX || cache_rows > INT32_MAX) return KD_EINVAL;
  return KD_OK;
}

// Both entry points: a contiguous cache (page_table == nullptr; cache rows B * cap) or a
// paged one (cache rows num_pages * page_size, cap = pages_per_req * page_size).
// `clear_ws` zeroes the workspace's control block and split tickets (after every
// check, right before the launch).
static int verify_attn_impl(const kd_bf16_t* q_abs, const kd_bf16_t* q_rope, const kd_bf16_t* c_kv,
                            const kd_bf16_t* k_rope, int64_t sc, int64_t sr, int64_t cap,
                            const int32_t* cache_lens, const uint32_t* vis, const int32_t* positions,
                            int B, int n, int H, float scale, kd_bf16_t* out, float* lse,
                            void* workspace, size_t ws_bytes, int kv_splits, const int32_t* page_table,
                            int page_size, int64_t pages_per_req, int64_t num_pages, bool clear_ws,
                            cudaStream_t stream) {
  const bool paged = page_table != nullptr;
  const int64_t cache_rows = paged ? num_pages * page_size : (int64_t)B * cap;
  int st = check_attn_args(q_abs, q_rope, c_kv, k_rope, sc, sr, cap, cache_lens, vis, B, n, H, scale, out,
                           lse, kv_splits, cache_rows);
  if (st) return st;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return KD_EINVAL;
  const int64_t rows = (int64_t)B * n * H;
  int sms = 0;
  if ((st = device_sms(&sms))) return st;
  static std::once_flag attr_once[64];
  static std::atomic<int> attr_status[64];
  int dev = 0;
  if ((st = cuda_status(cudaGetDevice(&dev), "cudaGetDevice"))) return st;
  if (dev < 0 || dev >= 64) return KD_ENODEV;
  std::call_once(attr_once[dev], [&] {
    int s = cuda_status(cudaFuncSetAttribute(tc::attn_tc_kernel<false>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, tc::SMEM_BYTES),
                        "cudaFuncSetAttribute(attn_tc_kernel)");
    if (!s)
      s = cuda_status(cudaFuncSetAttribute(tc::attn_tc_kernel<true>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, tc::SMEM_BYTES),
                      "cudaFuncSetAttribute(attn_tc_kernel, paged)");
    attr_status[dev].store(s);
  });
  if ((st = attr_status[dev].load())) return st;
  const int pairs = tc::active_pairs(sms);
  int splits = kv_splits;
  if (splits == 0) {
    // the automatic choice, lowered until its partials fit the workspace given
    splits = auto_splits(B, n, H, cap, pairs);
    while (splits > 1 && workspace_bytes_for(B, n, H, splits) > ws_bytes) --splits;
  }
  if (workspace_bytes_for(B, n, H, splits) > ws_bytes) return KD_ERANGE;

  CUtensorMap tq, tr, tcv, tkr, tv;
  if ((st = tc::make_map(&tq, q_abs, KD_D_C, (uint64_t)rows, KD_D_C * 2, tc::BM))) return st;
  if ((st = tc::make_map(&tr, q_rope, KD_D_R, (uint64_t)rows, KD_D_R * 2, tc::BM))) return st;
  const uint32_t kbox = paged ? (uint32_t)page_size : (uint32_t)tc::BQ;    // K box rows (one page)
  if ((st = tc::make_map(&tcv, c_kv, KD_D_C, (uint64_t)cache_rows, (uint64_t)sc * 2, kbox))) return st;
  if ((st = tc::make_map(&tkr, k_rope, KD_D_R, (uint64_t)cache_rows, (uint64_t)sr * 2, kbox))) return st;
  if ((st = tc::make_map(&tv, c_kv, KD_D_C, (uint64_t)cache_rows, (uint64_t)sc * 2, tc::VKEYS))) return st;

  const WsLayout wl = ws_layout(B, n, H, splits);
  tc::Params prm;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  prm.cache_lens = cache_lens;
  prm.vis = vis;
  prm.positions = positions;
  prm.out = out;
  prm.lse = lse;
  prm.err = reinterpret_cast<int32_t*>(ws);
  prm.sched = reinterpret_cast<unsigned long long*>(ws + 8);
  prm.tickets = splits > 1 ? reinterpret_cast<int32_t*>(ws + wl.tickets) : nullptr;
  prm.part_lse = splits > 1 ? reinterpret_cast<float*>(ws + wl.part_lse) : nullptr;
  prm.part_o = splits > 1 ? reinterpret_cast<float*>(ws + wl.part_o) : nullptr;
  prm.cap = cap;
  prm.B = B;
  prm.n = n;
  prm.H = H;
  prm.W = (n + 31) / 32;
  prm.mtiles = (int)((rows / B + tc::BM - 1) / tc::BM);
  prm.splits = splits;
  prm.units = (int64_t)B * prm.mtiles * splits;
  if (prm.units > INT32_MAX) return KD_EINVAL;     // unit ranks are 32-bit on the device
  prm.clusters = (int)(prm.units < pairs ? prm.units : pairs);
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.page_table = page_table;
  prm.page_size = paged ? page_size : 1;
  prm.page_shift = paged ? (page_size == 64 ? 6 : page_size == 128 ? 7 : 8) : 0;
  prm.pages_per_req = paged ? (int)pages_per_req : 0;
  prm.num_pages = paged ? num_pages : 0;
  CUtensorMap to;
  if ((st = splits > 1 ? tc::make_out_map(&to, prm.part_o, true, (uint64_t)(rows / B), (uint64_t)splits * B)
                       : tc::make_out_map(&to, out, false, (uint64_t)(rows / B), (uint64_t)B)))
    return st;
  if (clear_ws && (st = cuda_status(cudaMemsetAsync(workspace, 0, splits > 1 ? wl.part_lse : 256, stream),
                                    "cudaMemsetAsync(workspace)")))
    return st;
  const dim3 grid((unsigned)(2 * prm.clusters));
  if (paged)
    tc::attn_tc_kernel<true><<<grid, tc::NTHREADS, tc::SMEM_BYTES, stream>>>(tq, tr, tcv, tkr, tv, to, prm);
  else
    tc::attn_tc_kernel<false><<<grid, tc::NTHREADS, tc::SMEM_BYTES, stream>>>(tq, tr, tcv, tkr, tv, to, prm);
  return launch_status("attn_tc_kernel");
}

extern "C" int kd_tree_verify_attn(const kd_bf16_t* q_abs, const kd_bf16_t* q_rope,
                                   const kd_bf16_t* c_kv, const kd_bf16_t* k_rope, int64_t sc,
                                   int64_t sr, int64_t cap, const int32_t* cache_lens,
                                   const uint32_t* vis, const int32_t* positions, int B, int n,
                                   int H, float scale, kd_bf16_t* out, float* lse, void* workspace,
                                   size_t ws_bytes, int kv_splits, cudaStream_t stream) {
  return verify_attn_impl(q_abs, q_rope, c_kv, k_rope, sc, sr, cap, cache_lens, vis, positions, B, n,
                          H, scale, out, lse, workspace, ws_bytes, kv_splits, nullptr, 1, 0, 0, false, stream);
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
                          kv_splits, page_table, page_size, pages_per_req, num_pages, false, stream);
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
  // every argument is checked before anything is enqueued
  int st = check_attn_args(q_nope_absorbed, q_rope, c_kv, k_rope, kv_row_stride_c, kv_row_stride_r, cap,
                           cache_lens, vis, B, n, H, scale, out, lse, kv_splits, (int64_t)B * cap);
  if (st) return st;
  // Requests that need more split-KV scratch than the array holds are refused here;
  // with kv_splits = 0 the automatic policy picks a split count that fits.
  if (kv_splits > 0 && workspace_bytes_for(B, n, H, kv_splits) > (size_t)KD_NOALLOC_SCRATCH_BYTES)
    return KD_ERANGE;
  // Host code sees the array's name only as a stand-in, so the device address is
  // looked up once per device, with that device current, on the first call.
  static std::once_flag once[64];
  static std::atomic<void*> scratch_ptr[64];
  static std::atomic<int> lookup_status[64];
  int dev = 0;
  if ((st = cuda_status(cudaGetDevice(&dev), "cudaGetDevice"))) return st;
  if (dev < 0 || dev >= 64) return KD_ENODEV;
  std::call_once(once[dev], [&] {
    void* ptr = nullptr;
    const int s = cuda_status(cudaGetSymbolAddress(&ptr, kd::g_noalloc_scratch), "cudaGetSymbolAddress");
    scratch_ptr[dev].store(s ? nullptr : ptr);
    lookup_status[dev].store(s);
  });
  if ((st = lookup_status[dev].load())) return st;
  void* scratch = scratch_ptr[dev].load();
  // the control block and the split tickets start at zero on every call
  st = verify_attn_impl(q_nope_absorbed, q_rope, c_kv, k_rope, kv_row_stride_c, kv_row_stride_r, cap,
                        cache_lens, vis, positions, B, n, H, scale, out, lse, scratch,
                        (size_t)KD_NOALLOC_SCRATCH_BYTES, kv_splits, nullptr, 1, 0, 0, true, stream);
  if (st) return st;
  if (dev_error)
    st = cuda_status(cudaMemcpyAsync(dev_error, scratch, sizeof(int32_t), cudaMemcpyDeviceToDevice, stream),
                     "cudaMemcpyAsync(error word)");
  return st;
}
