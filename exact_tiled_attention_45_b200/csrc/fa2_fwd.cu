// Exact attention forward for B200 (sm_100a): tiled, online softmax, tcgen05
// tensor-core MMAs accumulating in tensor memory, TMA tile loads, and
// warp-specialised roles.
//
// Method (FlashAttention-2, Tri Dao, arXiv 2307.08691):
//  * arXiv abstract page, "Abstract" (1)-(3) and iplexlaw blog "FlashAttention-2:
//    making long-context attention run efficiently on GPUs", section "Three
//    changes improve GPU utilisation":
//      (1) fewer non-matmul FLOPs: the running max/sum live in registers, the
//          1/l normalisation is deferred to the epilogue, exponentials use exp2
//          with the softmax scale folded into one FMA, and only the diagonal
//          (causal) or ragged tail tile is masked element by element;
//      (2) parallel over the sequence: one CTA per (256-row query block, head,
//          batch); with causal masking the blocks of a group of heads launch
//          heaviest first;
//      (3) work split without shared-memory reductions: each softmax thread
//          owns one query row (one TMEM lane) from scores to output.
//  * iplexlaw blog, section "Tiling preserves the attention calculation":
//    K/V are streamed through on-chip memory tile by tile; the online softmax
//    rescales partial outputs so the result is the globally normalised one.
//
// B200 design (not in the pages, which describe A100 kernels):
//  * a CTA owns two 128-row query tiles (t = 0, 1) that share every K/V tile;
//    the tensor core works on one tile while the softmax warpgroup of the
//    other tile computes exponentials (ping-pong);
//  * warp 8 = TMA producer (Q0, Q1 once; K and V through separate rings);
//  * warp 9 = MMA issuer.  Per K/V tile j it issues
//        PV_0(j-1), S_0(j), PV_1(j-1), S_1(j)
//    with S_t = Q_t K_j^T (both operands in shared memory) into tile t's TMEM
//    score columns and O_t += P_t V (P read from TMEM, V from shared memory);
//  * warpgroup t (warps 4t..4t+3) = softmax of tile t: thread r <-> query row
//    r <-> TMEM lane r.  P (bf16) is written over the first 64 score columns;
//  * the O rescale is skipped unless a row's running max grows by more than
//    RESCALE_THRESHOLD (log2 units).  The stale max is used consistently for
//    P, the running sum and the final LSE, so the result is unchanged (the
//    exponentials stay below 2^RESCALE_THRESHOLD);
//  * every wait is bounded; on time-out the kernel records a status word,
//    drains its own in-flight copies and MMAs, frees TMEM and returns.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "fa2.h"
#include "sm100_ptx.cuh"

namespace fa2 {

using namespace ptx;

constexpr int BM = 128;         // query rows per tile (one tcgen05 M=128 MMA)
constexpr int Q_TILES = 2;      // query tiles per CTA
constexpr int BLOCK_M = BM * Q_TILES;
constexpr int BN = 128;         // keys per K/V tile
constexpr int NUM_THREADS = 384;
constexpr int PRODUCER_WARP = 8;
constexpr int MMA_WARP = 9;
constexpr uint32_t TMEM_COLS = 512;
// TMEM columns of tile t: scores at 128*t (P aliases the first 64 of them),
// output accumulator at 256 + 128*t.
__host__ __device__ constexpr uint32_t tm_s(int t) { return 128u * static_cast<uint32_t>(t); }
__host__ __device__ constexpr uint32_t tm_o(int t) { return 256u + 128u * static_cast<uint32_t>(t); }
constexpr float RESCALE_THRESHOLD = 8.0f;
#ifndef FA2_EMU_PAIRS_D128
#define FA2_EMU_PAIRS_D128 1
#endif
#ifndef FA2_EMU_PAIRS_D64
#define FA2_EMU_PAIRS_D64 3
#endif
// Register split: launched at 168 per thread (384 threads), the softmax
// warpgroups grow to 216 and the control warpgroup shrinks to 72:
// 256*216 + 128*72 = 64512 <= 384*168 = 64512.
constexpr uint32_t REGS_SOFTMAX = 216;
constexpr uint32_t REGS_CONTROL = 72;
static_assert(256 * REGS_SOFTMAX + 128 * REGS_CONTROL <= 384 * 168, "register split exceeds the launch budget");

// Optional per-role timeline (compile with -DFA2_TRACE): SM clock stamps of
// the pipeline events of CTA (0,0,0), read back with fa2_trace_read().  The
// product build compiles every stamp away.
#ifdef FA2_TRACE
constexpr int TRACE_J = 64;   // K/V tiles recorded
constexpr int TRACE_EV = 32;  // event kinds
__device__ long long g_fa2_trace[TRACE_EV * TRACE_J + 1];
#define FA2_STAMP(ev, j)                                                                          \
  do {                                                                                            \
    if (blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0 && (j) >= 0 && (j) < TRACE_J)        \
      g_fa2_trace[(ev) * TRACE_J + (j)] = clock64();                                              \
  } while (0)
#else
#define FA2_STAMP(ev, j) \
  do {                   \
  } while (0)
#endif

// Device status word: bit 0 = a bounded wait gave up; bits 8..11 = role.
__device__ unsigned int g_fa2_status = 0;
constexpr unsigned int STATUS_TIMEOUT = 1u;
constexpr unsigned int ROLE_PRODUCER = 1u << 8, ROLE_MMA = 2u << 8, ROLE_SOFTMAX = 3u << 8,
                       ROLE_DRAIN = 4u << 8;

template <int HD>
struct Cfg {
  static_assert(HD == 64 || HD == 128, "head dimension");
  static constexpr int KCH = HD / 64;                   // 64-element (128-byte) column chunks
  static constexpr int CHUNK_BYTES = 128 * 128;         // 128 rows x 128 bytes
  static constexpr int TILE_BYTES = KCH * CHUNK_BYTES;  // one 128-row Q/K/V tile
  static constexpr int KS = (HD == 128) ? 2 : 3;        // K ring stages
  static constexpr int VS = (HD == 128) ? 2 : 3;        // V ring stages
  // Of every 8 pairs of scores, this many are exponentiated on the FMA pipe
  // (polynomial) and the rest on the special-function unit.  At d = 128 the
  // special-function work of a tile equals its MMA time; at d = 64 it is twice.
  static constexpr int EMU_PAIRS_PER_8 = (HD == 128) ? FA2_EMU_PAIRS_D128 : FA2_EMU_PAIRS_D64;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_TILES * TILE_BYTES;
  static constexpr int OFF_V = OFF_K + KS * TILE_BYTES;
  static constexpr int OFF_BAR = OFF_V + VS * TILE_BYTES;
  static constexpr int SMEM_BYTES = OFF_BAR + 256 + 1024;  // barriers + alignment slack
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

struct Params {
  __nv_bfloat16* o;
  float* lse;
  int N;
  int BH;           // B * H
  int n_q_blocks;   // 256-row query blocks
  int n_kv_tiles;   // 128-key tiles
  int group_heads;  // heads per launch-order group (see the kernel's work mapping)
  float scale_log2;  // scale * log2(e)
  unsigned long long timeout_ns;
  int inject_timeout;  // test hook: withhold the Q loads
};

struct Barriers {
  uint64_t q_full[2];
  uint64_t k_full[3], k_empty[3];
  uint64_t v_full[3], v_empty[3];
  uint64_t s_full[2];   // S_t(j) complete (and every MMA issued before it)
  uint64_t p_full[2];   // softmax t wrote P_t(j) (and rescaled O_t if needed)
  uint64_t o_ready[2];  // last PV_t complete
  uint64_t mma_final[2];
  uint64_t epi[2];      // the four warps of softmax group t wrote their O rows to shared memory
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(Barriers) <= 256, "barrier block");

// Bounded wait.  Returns false (and records the time-out once) if the phase
// did not complete within timeout_ns, or if another role already gave up.
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                             unsigned long long timeout_ns, unsigned int role) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > timeout_ns) {
      *abort_flag = 1;
      atomicOr(&g_fa2_status, STATUS_TIMEOUT | role);
      return false;
    }
  }
}

// Warp-uniform bounded wait for the softmax warps (all 32 lanes agree).
__device__ __forceinline__ bool wait_warp(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          unsigned long long timeout_ns) {
  const bool ok = wait_bounded(bar, parity, abort_flag, timeout_ns, ROLE_SOFTMAX);
  return __all_sync(0xffffffffu, ok);
}

// Bounded wait used while draining: ignores the abort flag.
__device__ __forceinline__ bool wait_drain(uint32_t bar, uint32_t parity, unsigned long long timeout_ns) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > timeout_ns) {
      atomicOr(&g_fa2_status, STATUS_TIMEOUT | ROLE_DRAIN);
      return false;
    }
  }
  return true;
}

// Number of K/V tiles query tile t of block qb attends to.
template <bool CAUSAL>
__device__ __forceinline__ int kv_tiles_for(int qb, int t, int n_kv_tiles) {
  if (!CAUSAL) return n_kv_tiles;
  return min(qb * Q_TILES + t + 1, n_kv_tiles);  // the diagonal tile is the last one
}

// ------------------------------------------------------------------ softmax
// One thread = one query row of tile t.  Returns false if a wait gave up.
template <int HD, bool CAUSAL>
__device__ __forceinline__ void softmax_role(const Params& p, const CUtensorMap* tmap_o, uint32_t sQt, Barriers* bars,
                                             volatile int* abort_flag, uint32_t tmem, int t, int warp_in_wg, int lane,
                                             int row_g, int bh, int n_t) {
  const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp_in_wg * 32) << 16);
  const uint32_t s_addr = lane_base + tm_s(t);
  const uint32_t o_addr = lane_base + tm_o(t);
  const uint32_t b_s = smem_u32(&bars->s_full[t]);
  const uint32_t b_p = smem_u32(&bars->p_full[t]);
  const float c_log2 = p.scale_log2;
  const uint64_t cc = f2_pack(c_log2, c_log2);
  const int q_first = row_g - (warp_in_wg * 32 + lane);  // first row of this tile
  float m = -INFINITY;  // running max of scale*log2(e)*s (possibly stale, see header)
  float l = 0.f;        // running sum of exp2(...) relative to m
  bool ok = true;
  for (int j = 0; j < n_t; ++j) {
    ok = wait_warp(b_s, j & 1, abort_flag, p.timeout_ns);
    if (!ok) break;
    if (lane == 0 && warp_in_wg < 2) FA2_STAMP(warp_in_wg == 0 ? 12 + 6 * t : 22 + t, j);
    tc_fence_after();
    uint32_t s[128];
#pragma unroll
    for (int c = 0; c < 4; ++c) tmem_ld32(s_addr + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&s[c * 32]));
    tmem_wait_ld();
#pragma unroll
    for (int c = 0; c < 4; ++c) reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(&s[c * 32]));

    const int kv0 = j * BN;
    const bool diag = CAUSAL && (kv0 + BN - 1 > q_first);  // tile reaches past this tile's first row
    const bool tail = !CAUSAL && (kv0 + BN > p.N);          // ragged last key tile
    if (diag || tail) {
      const int lim = diag ? (row_g - kv0) : (p.N - 1 - kv0);  // last allowed column
#pragma unroll
      for (int e = 0; e < 128; ++e)
        if (e > lim) s[e] = __float_as_uint(-INFINITY);
    }
    // Row max: eight independent chains (3-input max over columns 8..119,
    // then columns 120..127), then combine.
    float mx8[8];
#pragma unroll
    for (int a = 0; a < 8; ++a) mx8[a] = __uint_as_float(s[a]);
#pragma unroll
    for (int e = 8; e + 16 <= 128; e += 16)
#pragma unroll
      for (int a = 0; a < 8; ++a) mx8[a] = fmax3(mx8[a], __uint_as_float(s[e + a]), __uint_as_float(s[e + 8 + a]));
#pragma unroll
    for (int a = 0; a < 8; ++a) mx8[a] = fmaxf(mx8[a], __uint_as_float(s[120 + a]));
    const float mx = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]));
    const float m_cand = mx * c_log2;
    float m_new = m;
    if (m_cand > m + RESCALE_THRESHOLD) m_new = m_cand;  // also taken on the first tile (m = -inf)
    const bool rescale = (j > 0) && (m_new != m);
    const float alpha = rescale ? ex2(m - m_new) : 1.f;
    const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
    const uint64_t mm = f2_pack(-m_use, -m_use);

    // p = exp2(s*c - m): one packed FMA per pair, ex2 per element; P packed to
    // bf16 and written over the score columns 32 at a time.
    uint64_t acc[4] = {0, 0, 0, 0};
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t pk[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const int i = h * 64 + 2 * e;
        const uint64_t x = f2_fma(f2_pack(__uint_as_float(s[i]), __uint_as_float(s[i + 1])), cc, mm);
        float p0, p1;
        if (((h * 32 + e) & 7) < Cfg<HD>::EMU_PAIRS_PER_8) {
          f2_unpack(exp2_poly_pair(x), p0, p1);  // FMA pipe
        } else {
          float x0, x1;
          f2_unpack(x, x0, x1);
          p0 = ex2(x0);  // special-function unit
          p1 = ex2(x1);
        }
        acc[e & 3] = f2_add(acc[e & 3], f2_pack(p0, p1));
        pk[e] = pack_bf16x2(p0, p1);
      }
      tmem_st32(s_addr + h * 32, pk);
    }
    float r0, r1, r2, r3, r4, r5, r6, r7;
    f2_unpack(f2_add(acc[0], acc[1]), r0, r1);
    f2_unpack(f2_add(acc[2], acc[3]), r2, r3);
    (void)r4; (void)r5; (void)r6; (void)r7;
    const float rowsum = (r0 + r1) + (r2 + r3);

    // S_t(j) complete implies PV_t(j-1) complete (the commit tracks every
    // earlier MMA), so O_t is stable here.
    if (warp_in_wg == 0 && lane == 0) FA2_STAMP(13 + 6 * t, j);
    if (__any_sync(0xffffffffu, rescale)) {
      const uint64_t aa = f2_pack(alpha, alpha);
#pragma unroll
      for (int c = 0; c < HD / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(o_addr + c * 32, o);
        tmem_wait_ld();
        reg_fence32(o);
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          float a0, a1;
          f2_unpack(f2_mul(f2_pack(__uint_as_float(o[e]), __uint_as_float(o[e + 1])), aa), a0, a1);
          o[e] = __float_as_uint(a0);
          o[e + 1] = __float_as_uint(a1);
        }
        tmem_st32(o_addr + c * 32, o);
      }
    }
    tmem_wait_st();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(b_p);
    if (lane == 0) FA2_STAMP(8 + 6 * t + warp_in_wg, j);
    l = l * alpha + rowsum;
    m = m_new;
  }
  if (ok) ok = wait_warp(smem_u32(&bars->o_ready[t]), 0, abort_flag, p.timeout_ns);
  if (!ok) return;
  if (warp_in_wg == 0 && lane == 0) FA2_STAMP(24 + t, 0);
  tc_fence_after();
  // Epilogue: O / l in bf16 is written into this tile's Q buffer (free: the
  // o_ready commit tracks the tile's last S MMA) in the 128-byte-swizzled
  // layout of the O tensor map, then one thread stores the tile with TMA.
  const float inv_l = (l > 0.f) ? 1.f / l : 0.f;
  const bool store = row_g < p.N;
  const int r = warp_in_wg * 32 + lane;
  const uint64_t il = f2_pack(inv_l, inv_l);
  uint32_t o[HD / 32][32];
#pragma unroll
  for (int c = 0; c < HD / 32; ++c) tmem_ld32(o_addr + c * 32, o[c]);
  tmem_wait_ld();
#pragma unroll
  for (int c = 0; c < HD / 32; ++c) reg_fence32(o[c]);
#pragma unroll
  for (int c = 0; c < HD / 32; ++c) {
    uint32_t w[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      float a0, a1;
      f2_unpack(f2_mul(f2_pack(__uint_as_float(o[c][2 * e]), __uint_as_float(o[c][2 * e + 1])), il), a0, a1);
      w[e] = pack_bf16x2(a0, a1);
    }
    // 32 columns = 64 bytes = four 16-byte pieces of the row's 128-byte line
    // in 64-column chunk c/2; piece k sits at (k ^ (r % 8)) * 16.
    const uint32_t line = sQt + (c >> 1) * (128 * 128) + r * 128;
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const int k = (c & 1) * 4 + v;
      st_shared_v4(line + ((k ^ (r & 7)) << 4), w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
    }
  }
  // Every warp's rows are in shared memory before the store is issued; only
  // the storing thread waits (bounded), so a warp that gave up earlier cannot
  // leave the others blocked.
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) mbar_arrive(smem_u32(&bars->epi[t]));
  const int tile_row0 = row_g - r;
  if (warp_in_wg == 0 && lane == 0 && tile_row0 < p.N &&
      wait_bounded(smem_u32(&bars->epi[t]), 0, abort_flag, p.timeout_ns, ROLE_SOFTMAX)) {
#pragma unroll
    for (int c = 0; c < HD / 64; ++c) tma_store_3d(tmap_o, sQt + c * (128 * 128), c * 64, tile_row0, bh);
    bulk_commit_group();
    bulk_wait_read();  // the shared-memory source must stay valid until read
  }
  if (store) {
    const float lse = (l > 0.f) ? (m + log2f(l)) * 0.69314718055994531f : -INFINITY;
    p.lse[static_cast<size_t>(bh) * p.N + row_g] = lse;
  }
  if (warp_in_wg == 0 && lane == 0) FA2_STAMP(26 + t, 0);
}

template <int HD, bool CAUSAL>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    fa2_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_out,
                   const Params p) {
  using C = Cfg<HD>;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte alignment for the 128-byte-swizzle atoms.
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t base = (raw_addr + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw_addr);
  Barriers* bars = reinterpret_cast<Barriers*>(smem + C::OFF_BAR);
  volatile int* abort_flag = &bars->abort;

  const uint32_t sQ = base + C::OFF_Q;
  const uint32_t sK = base + C::OFF_K;
  const uint32_t sV = base + C::OFF_V;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // Work mapping of the 1-D grid (CTAs launch roughly in index order): the
  // heads are taken in groups of group_heads; within a group the query-block
  // rank is the slow index and the head the fast one.  With causal masking
  // rank 0 is the heaviest block, so each group runs longest-first and the
  // last wave holds the lightest blocks; a group's K/V stays small enough to
  // be reused from L2 by its blocks.  Without masking every block costs the
  // same and group_heads = 1 (all blocks of a head in a row).
  const int per_group = p.group_heads * p.n_q_blocks;
  const int grp = static_cast<int>(blockIdx.x) / per_group;
  const int in_grp = static_cast<int>(blockIdx.x) - grp * per_group;
  const int grp_heads = min(p.group_heads, p.BH - grp * p.group_heads);
  const int rank = in_grp / grp_heads;
  const int bh = grp * p.group_heads + (in_grp - rank * grp_heads);
  const int qb = CAUSAL ? (p.n_q_blocks - 1 - rank) : rank;
  const int q0 = qb * BLOCK_M;
  const int n0 = kv_tiles_for<CAUSAL>(qb, 0, p.n_kv_tiles);
  const int n1 = kv_tiles_for<CAUSAL>(qb, 1, p.n_kv_tiles);  // n0 <= n1

  if (threadIdx.x == 0) {
    for (int t = 0; t < 2; ++t) {
      mbar_init(smem_u32(&bars->q_full[t]), 1);
      mbar_init(smem_u32(&bars->s_full[t]), 1);
      mbar_init(smem_u32(&bars->p_full[t]), 4);
      mbar_init(smem_u32(&bars->o_ready[t]), 1);
    }
    for (int s = 0; s < C::KS; ++s) {
      mbar_init(smem_u32(&bars->k_full[s]), 1);
      mbar_init(smem_u32(&bars->k_empty[s]), 1);
    }
    for (int s = 0; s < C::VS; ++s) {
      mbar_init(smem_u32(&bars->v_full[s]), 1);
      mbar_init(smem_u32(&bars->v_empty[s]), 1);
    }
    mbar_init(smem_u32(&bars->mma_final[0]), 1);
    mbar_init(smem_u32(&bars->mma_final[1]), 1);
    mbar_init(smem_u32(&bars->epi[0]), 4);
    mbar_init(smem_u32(&bars->epi[1]), 4);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == MMA_WARP) {
    tmem_alloc(smem_u32(&bars->tmem_base), TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == PRODUCER_WARP && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    prefetch_tmap(&tm_out);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
#ifdef FA2_TRACE
  if (threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0)
    g_fa2_trace[TRACE_EV * TRACE_J] = clock64();
#endif

  if (warp >= 8) {
    regs_dec<REGS_CONTROL>();
    if (warp == PRODUCER_WARP && lane == 0) {
      // ---------------------------------------------------------- TMA producer
      const bool load_q = !p.inject_timeout;
      // Q_0, K_0, Q_1, V_0, then K and V: the order the first MMAs need them.
      auto load_q_tile = [&](int t) {
        // A tile that starts at or past N has no row to store; it is loaded
        // from tile 0's rows so that no copy lies wholly outside the tensor.
        const int qy = (q0 + t * BM < p.N) ? q0 + t * BM : q0;
        const uint32_t qbar = smem_u32(&bars->q_full[t]);
        mbar_arrive_expect_tx(qbar, C::TILE_BYTES);
        for (int c = 0; c < C::KCH; ++c)
          tma_load_3d(sQ + t * C::TILE_BYTES + c * C::CHUNK_BYTES, &tm_q, qbar, c * 64, qy, bh);
      };
      if (load_q) load_q_tile(0);
      int k_issued = 0, v_issued = 0;
      for (int j = 0; j < n1; ++j) {
        const int ks = j % C::KS;
        if (j >= C::KS &&
            !wait_bounded(smem_u32(&bars->k_empty[ks]), ((j / C::KS) - 1) & 1, abort_flag, p.timeout_ns,
                          ROLE_PRODUCER))
          break;
        const uint32_t kb = smem_u32(&bars->k_full[ks]);
        FA2_STAMP(20, j);
        mbar_arrive_expect_tx(kb, C::TILE_BYTES);
        for (int c = 0; c < C::KCH; ++c)
          tma_load_3d(sK + ks * C::TILE_BYTES + c * C::CHUNK_BYTES, &tm_k, kb, c * 64, j * BN, bh);
        ++k_issued;
        if (j == 0 && load_q) load_q_tile(1);
        const int vs = j % C::VS;
        if (j >= C::VS &&
            !wait_bounded(smem_u32(&bars->v_empty[vs]), ((j / C::VS) - 1) & 1, abort_flag, p.timeout_ns,
                          ROLE_PRODUCER))
          break;
        const uint32_t vb = smem_u32(&bars->v_full[vs]);
        FA2_STAMP(21, j);
        mbar_arrive_expect_tx(vb, C::TILE_BYTES);
        for (int c = 0; c < C::KCH; ++c)
          tma_load_3d(sV + vs * C::TILE_BYTES + c * C::CHUNK_BYTES, &tm_v, vb, c * 64, j * BN, bh);
        ++v_issued;
      }
      // Drain: every load this thread issued must land before the CTA exits.
      if (load_q) {
        wait_drain(smem_u32(&bars->q_full[0]), 0, p.timeout_ns);
        wait_drain(smem_u32(&bars->q_full[1]), 0, p.timeout_ns);
      }
      for (int t = (k_issued > C::KS ? k_issued - C::KS : 0); t < k_issued; ++t)
        wait_drain(smem_u32(&bars->k_full[t % C::KS]), (t / C::KS) & 1, p.timeout_ns);
      for (int t = (v_issued > C::VS ? v_issued - C::VS : 0); t < v_issued; ++t)
        wait_drain(smem_u32(&bars->v_full[t % C::VS]), (t / C::VS) & 1, p.timeout_ns);
    } else if (warp == MMA_WARP && lane == 0) {
      // ---------------------------------------------------------- MMA issuer
      // The tensor pipe keeps about one MMA queued, so any wait or commit
      // between two MMAs longer than one MMA (64 cycles) is idle pipe time.
      // Only the softmax hand-offs are waited for between groups; the K/V
      // waits run under the MMAs of the preceding group where possible.
      constexpr uint32_t IDESC_S = idesc_bf16_f32(BM, BN, false, false);
      constexpr uint32_t IDESC_PV = idesc_bf16_f32(BM, HD, false, true);
      // `hook` runs after the second MMA of a group: a wait placed there
      // overlaps the MMA the pipe is executing instead of idling it.
      auto issue_s = [&](int t, int ks, auto&& hook) {
        const uint32_t qbase = sQ + t * C::TILE_BYTES;
        const uint32_t kbase = sK + ks * C::TILE_BYTES;
        const uint32_t d_s = tmem + tm_s(t);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::CHUNK_BYTES + (kk & 3) * 32;
          mma_ss(d_s, smem_desc_sw128(qbase + off, 16, 1024), smem_desc_sw128(kbase + off, 16, 1024), IDESC_S,
                 kk > 0 ? 1u : 0u);
          if (kk == 1) hook();
        }
      };
      auto issue_pv = [&](int t, int vs, bool acc, auto&& hook) {
        const uint32_t vbase = sV + vs * C::TILE_BYTES;
        const uint32_t d_o = tmem + tm_o(t), a_p = tmem + tm_s(t);
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          mma_ts(d_o, a_p + kk * 8, smem_desc_sw128(vbase + kk * 2048, C::CHUNK_BYTES, 1024), IDESC_PV,
                 (acc || kk > 0) ? 1u : 0u);
          if (kk == 1) hook();
        }
      };
      const unsigned long long to = p.timeout_ns;
      bool ok = true;
      auto wait = [&](const uint64_t* bar, uint32_t parity) {
        ok = ok && wait_bounded(smem_u32(bar), parity, abort_flag, to, ROLE_MMA);
      };
      auto nothing = [] {};
      // K/V tile 0: S_0(0), S_1(0); Q_1 (and V_0 with a 3-stage V ring) are
      // waited for under the MMAs.
      wait(&bars->q_full[0], 0);
      wait(&bars->k_full[0], 0);
      if (ok) {
        tc_fence_after();
        issue_s(0, 0, [&] { wait(&bars->q_full[1], 0); });
        mma_commit(smem_u32(&bars->s_full[0]));
        FA2_STAMP(3, 0);
      }
      if (ok) {
        issue_s(1, 0, [&] {
          if (C::VS >= 3) wait(&bars->v_full[0], 0);
        });
        mma_commit(smem_u32(&bars->s_full[1]));
        mma_commit(smem_u32(&bars->k_empty[0]));
        FA2_STAMP(7, 0);
      }
      // Step j: PV_0(j-1), S_0(j), PV_1(j-1), S_1(j).  Tile 0 may stop one
      // K/V tile earlier (causal diagonal).  K(j) is waited for under PV_0's
      // MMAs (PV_1's when tile 0 is done); with a 3-stage V ring V(j) is
      // waited for under PV_1's MMAs of step j, otherwise at step j+1's start.
      for (int j = 1; ok && j <= n1; ++j) {
        const int i = j - 1;
        const int vs = i % C::VS;
        const int ks = j % C::KS;
        const bool do0 = i < n0, more0 = j < n0, more1 = j < n1;
        auto wait_k = [&] {
          if (more1) wait(&bars->k_full[ks], (j / C::KS) & 1);
        };
        FA2_STAMP(0, i);
        // V(j-1) from a 2-stage ring is waited for here, before the softmax
        // hand-off (usually the later of the two), so its latency overlaps
        // the softmax.
        if (C::VS < 3) wait(&bars->v_full[vs], (i / C::VS) & 1);
        if (do0) {
          wait(&bars->p_full[0], i & 1);
          if (!ok) break;
          FA2_STAMP(1, i);
          tc_fence_after();
          issue_pv(0, vs, i > 0, wait_k);
          FA2_STAMP(2, i);
          if (!ok) break;
          if (more0) issue_s(0, ks, nothing);
          mma_commit(smem_u32(more0 ? &bars->s_full[0] : &bars->o_ready[0]));
          FA2_STAMP(3, j);
        }
        FA2_STAMP(4, i);
        wait(&bars->p_full[1], i & 1);
        if (!ok) break;
        FA2_STAMP(5, i);
        tc_fence_after();
        issue_pv(1, vs, i > 0, [&] {
          if (!do0) wait_k();
          if (C::VS >= 3 && more1) wait(&bars->v_full[j % C::VS], (j / C::VS) & 1);
        });
        FA2_STAMP(6, i);
        if (!ok) break;
        if (more1) issue_s(1, ks, nothing);
        mma_commit(smem_u32(more1 ? &bars->s_full[1] : &bars->o_ready[1]));
        mma_commit(smem_u32(&bars->v_empty[vs]));
        if (more1) mma_commit(smem_u32(&bars->k_empty[ks]));
        FA2_STAMP(7, j);
      }
      // Drain: all MMAs issued by this thread complete before TMEM is freed.
      mma_commit(smem_u32(&bars->mma_final[0]));
      wait_drain(smem_u32(&bars->mma_final[0]), 0, p.timeout_ns);
    }
  } else {
    // ------------------------------------------------------------ softmax warpgroups
    regs_inc<REGS_SOFTMAX>();
    const int t = warp >> 2;            // query tile of this warpgroup
    const int warp_in_wg = warp & 3;    // TMEM lane quadrant
    const int r = warp_in_wg * 32 + lane;
    const int row_g = q0 + t * BM + r;
    softmax_role<HD, CAUSAL>(p, &tm_out, sQ + t * C::TILE_BYTES, bars, abort_flag, tmem, t, warp_in_wg, lane, row_g,
                             bh, t == 0 ? n0 : n1);
  }

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) FA2_STAMP(28, 0);
  if (warp == MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

#include "fa2_splitkv.cuh"
#include "fa2_bwd.cuh"

// ====================================================================== host

static thread_local char g_detail[512] = "";

static void set_detail(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_detail, sizeof(g_detail), fmt, ap);
  va_end(ap);
}

static PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn) return fn;
  void* ptr = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess)
    return nullptr;
  fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  return fn;
}

// View a [B*H, N, d] bf16 tensor as a 3-D TMA map with 64 x 128 x 1 boxes,
// 128-byte swizzle.  Rows past N read as zero.
static int make_tmap(CUtensorMap* tm, const void* ptr, int d, int N, int BH, int box_rows = 128) {
  auto enc = get_encode_fn();
  if (!enc) {
    set_detail("cuTensorMapEncodeTiled entry point unavailable");
    return FA2_ERR_CUDA;
  }
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(N) * d * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    set_detail("cuTensorMapEncodeTiled failed (CUresult %d)", static_cast<int>(r));
    return FA2_ERR_CUDA;
  }
  return FA2_OK;
}

// Streams and events of the host-buffer entry point, created once per device
// on first use and kept for the life of the process; the mutex serialises
// calls that share them (each call returns only after its work has landed).
struct HostPipe {
  static constexpr int MAX_CHUNKS = 8;
  std::mutex mu;
  cudaStream_t compute = nullptr, download = nullptr;
  cudaEvent_t uploaded[MAX_CHUNKS] = {}, computed[MAX_CHUNKS] = {}, drained = nullptr;
};

static int host_pipe(HostPipe** out) {
  constexpr int MAX_DEVICES = 64;
  static HostPipe pipes[MAX_DEVICES];
  static std::once_flag once[MAX_DEVICES];
  static int created[MAX_DEVICES] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) {
    set_detail("no usable current device");
    return FA2_ERR_CUDA;
  }
  std::call_once(once[dev], [dev] {
    HostPipe& p = pipes[dev];
    bool ok = cudaStreamCreateWithFlags(&p.compute, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&p.download, cudaStreamNonBlocking) == cudaSuccess &&
              cudaEventCreateWithFlags(&p.drained, cudaEventDisableTiming) == cudaSuccess;
    for (int i = 0; ok && i < HostPipe::MAX_CHUNKS; ++i)
      ok = cudaEventCreateWithFlags(&p.uploaded[i], cudaEventDisableTiming) == cudaSuccess &&
           cudaEventCreateWithFlags(&p.computed[i], cudaEventDisableTiming) == cudaSuccess;
    created[dev] = ok ? 1 : -1;
  });
  if (created[dev] != 1) {
    set_detail("could not create the host pipeline's streams and events");
    return FA2_ERR_CUDA;
  }
  *out = &pipes[dev];
  return FA2_OK;
}

static bool overlap(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

// Head dimensions served: 64 and 128 natively; 32 and 96 by the 64- and
// 128-column kernels, whose tiles TMA fills with zeros past d (loads) and
// clips at d (stores), so the padding adds nothing to S, P V or the outputs.
static bool d_supported(int d) { return d == 32 || d == 64 || d == 96 || d == 128 || d == 256; }
static int padded_hd(int d) { return d <= 64 ? 64 : (d <= 128 ? 128 : 256); }
// Keys per tile of the split-K/V kernel: 64 at d = 256, else 128.
static int skv_tile_keys(int d) { return padded_hd(d) == 256 ? 64 : 128; }

static int validate(const void* q, const void* k, const void* v, const void* o, const float* lse, int B, int H,
                    int N, int d, float scale) {
  if (!q || !k || !v || !o || !lse) {
    set_detail("null pointer");
    return FA2_ERR_INVALID_ARG;
  }
  if (B < 1 || H < 1 || N < 1 || B > 65535 || H > 65535 ||
      static_cast<long long>(B) * H * ((N + BLOCK_M - 1) / BLOCK_M) > 0x7fffffffLL) {
    set_detail("bad sizes B=%d H=%d N=%d (need B, H <= 65535 and B*H*ceil(N/256) < 2^31)", B, H, N);
    return FA2_ERR_INVALID_ARG;
  }
  if (!std::isfinite(scale) || !(scale > 0.f)) {
    set_detail("scale must be finite and positive");
    return FA2_ERR_INVALID_ARG;
  }
  if (!d_supported(d)) {
    set_detail("head dimension %d not supported (32, 64, 96, 128 or 256)", d);
    return FA2_ERR_UNSUPPORTED;
  }
  const uintptr_t mis = reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) |
                        reinterpret_cast<uintptr_t>(v) | reinterpret_cast<uintptr_t>(o);
  if ((mis & 15u) || (reinterpret_cast<uintptr_t>(lse) & 3u)) {
    set_detail("misaligned pointer (q/k/v/o need 16 bytes, lse 4)");
    return FA2_ERR_INVALID_ARG;
  }
  const size_t n_elem = static_cast<size_t>(B) * H * N * d;
  const size_t t_bytes = n_elem * 2, l_bytes = static_cast<size_t>(B) * H * N * 4;
  if (overlap(o, t_bytes, q, t_bytes) || overlap(o, t_bytes, k, t_bytes) || overlap(o, t_bytes, v, t_bytes) ||
      overlap(o, t_bytes, lse, l_bytes) || overlap(lse, l_bytes, q, t_bytes) ||
      overlap(lse, l_bytes, k, t_bytes) || overlap(lse, l_bytes, v, t_bytes)) {
    set_detail("output buffers overlap inputs or each other");
    return FA2_ERR_INVALID_ARG;
  }
  return FA2_OK;
}

template <int HD, bool CAUSAL>
static int launch_t(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& to,
                    const Params& prm, int B, int H, cudaStream_t stream) {
  using C = Cfg<HD>;
  auto kern = fa2_fwd_kernel<HD, CAUSAL>;
  static std::atomic<unsigned> attr_done_mask{0};  // per device bit (devices 0..31)
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    set_detail("cudaGetDevice failed");
    return FA2_ERR_CUDA;
  }
  if (dev >= 32 || !(attr_done_mask.load(std::memory_order_acquire) & (1u << dev))) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (e != cudaSuccess) {
      set_detail("cudaFuncSetAttribute: %s", cudaGetErrorString(e));
      return FA2_ERR_CUDA;
    }
    if (dev < 32) attr_done_mask.fetch_or(1u << dev, std::memory_order_acq_rel);
  }
  dim3 grid(B * H * prm.n_q_blocks);
  kern<<<grid, NUM_THREADS, C::SMEM_BYTES, stream>>>(tq, tk, tv, to, prm);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_detail("kernel launch: %s", cudaGetErrorString(e));
    return FA2_ERR_CUDA;
  }
  return FA2_OK;
}

static int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) == cudaSuccess && cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) ==
                                                 cudaSuccess && n > 0)
    return n;
  cudaGetLastError();  // no device here: plan for a B200
  return 148;
}

// Heads per launch-order group for causal masking: enough heads that the
// last group spans two waves of CTAs (so it can run longest-first), few
// enough that the group's K and V (4*N*d bytes per head) stay within 48 MiB
// of L2, then evened out over the groups.
static int causal_group_heads(int BH, int N, int d, int n_q_blocks) {
  const int sms = sm_count();
  int g = (2 * sms + n_q_blocks - 1) / n_q_blocks;
  const long long kv_head = 4LL * N * d;
  const long long g_l2 = std::max(1LL, (48LL << 20) / kv_head);
  g = static_cast<int>(std::min<long long>(std::min<long long>(g, g_l2), BH));
  const int groups = (BH + g - 1) / g;
  return (BH + groups - 1) / groups;
}

static int splitkv_impl(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Nq,
                        int Nk, int d, int causal, float scale, int n_splits, void* workspace,
                        size_t workspace_bytes, unsigned long long timeout_ns, int inject, cudaStream_t stream);

static int fwd_impl(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d,
                    int causal, float scale, unsigned long long timeout_ns, int inject, cudaStream_t stream) {
  g_detail[0] = 0;
  int st = validate(q, k, v, o, lse, B, H, N, d, scale);
  if (st != FA2_OK) return st;
  if (padded_hd(d) == 256) {
    // d = 256 runs on the one-tile kernel of the split-K/V path (64-key tiles)
    // as a single key range with Nq = Nk, which writes O and LSE directly.
    return splitkv_impl(q, k, v, o, lse, B, H, N, N, d, causal, scale, 1, nullptr, 0, timeout_ns, inject, stream);
  }
  CUtensorMap tq, tk, tv, to;
  const int BH = B * H;
  if ((st = make_tmap(&tq, q, d, N, BH)) != FA2_OK) return st;
  if ((st = make_tmap(&tk, k, d, N, BH)) != FA2_OK) return st;
  if ((st = make_tmap(&tv, v, d, N, BH)) != FA2_OK) return st;
  if ((st = make_tmap(&to, o, d, N, BH)) != FA2_OK) return st;
  Params prm;
  prm.o = static_cast<__nv_bfloat16*>(o);
  prm.lse = lse;
  prm.N = N;
  prm.BH = BH;
  prm.n_q_blocks = (N + BLOCK_M - 1) / BLOCK_M;
  prm.n_kv_tiles = (N + BN - 1) / BN;
  prm.group_heads = causal ? causal_group_heads(BH, N, d, prm.n_q_blocks) : 1;
  prm.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634074);
  prm.timeout_ns = timeout_ns;
  prm.inject_timeout = inject;
  if (padded_hd(d) == 64)
    return causal ? launch_t<64, true>(tq, tk, tv, to, prm, B, H, stream)
                  : launch_t<64, false>(tq, tk, tv, to, prm, B, H, stream);
  return causal ? launch_t<128, true>(tq, tk, tv, to, prm, B, H, stream)
                : launch_t<128, false>(tq, tk, tv, to, prm, B, H, stream);
}

constexpr unsigned long long DEFAULT_TIMEOUT_NS = 2000000000ull;  // 2 s per wait

// ------------------------------------------------------------------ split-K/V host side

constexpr int SKV_MAX_SPLITS = 128;

static bool skv_sizes_ok(int B, int H, int Nq, int Nk) {
  return B >= 1 && H >= 1 && Nq >= 1 && Nk >= Nq && static_cast<long long>(B) * H <= 65535;
}

// Number of key ranges actually used.  n_splits = 0 picks one: the work is a
// stream over K and V, so what matters is enough CTAs to keep most SMs
// loading; beyond that each extra range only adds set-up, partial writes and
// the merge.  So: the fewest ranges that give at least 0.8 x (SM count) CTAs,
// keeping at least 4 key tiles per range.  A requested count is capped at 128
// and at the number of key tiles, then reduced to ceil(tiles / ceil(tiles /
// s)) so that no range is empty by construction.
static int skv_resolve_splits(int B, int H, int Nq, int Nk, int n_splits, int tile_keys) {
  const int n_kv = (Nk + tile_keys - 1) / tile_keys;
  int s = n_splits;
  if (s <= 0) {
    const long long base = static_cast<long long>((Nq + BM - 1) / BM) * B * H;
    const long long want = (static_cast<long long>(sm_count()) * 4 + 4) / 5;
    s = base >= want ? 1 : static_cast<int>((want + base - 1) / base);
    s = std::max(1, std::min(s, n_kv / 4));
  }
  s = std::min(std::min(s, SKV_MAX_SPLITS), n_kv);
  const int tps = (n_kv + s - 1) / s;
  return (n_kv + tps - 1) / tps;
}

static size_t round256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Workspace layout: o_part fp32 [splits, B*H, Nq, d], then lse_part fp32
// [splits, B*H, Nq], each starting on a 256-byte boundary.  A single range
// needs none.
static size_t skv_workspace_bytes(int B, int H, int Nq, int d, int splits) {
  if (splits <= 1) return 0;
  const size_t rows = static_cast<size_t>(splits) * B * H * Nq;
  return round256(rows * d * 4) + round256(rows * 4);
}

template <int HD, bool CAUSAL, bool QUAD>
static int skv_launch_t(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const SkvParams& prm,
                        int n_q_tiles, int splits, __nv_bfloat16* o, float* lse, cudaStream_t stream) {
  using C = SkvCfg<HD, skv_slim<HD, QUAD>()>;
  auto kern = fa2_splitkv_kernel<HD, CAUSAL, QUAD>;
  static std::atomic<unsigned> attr_done_mask{0};  // per device bit (devices 0..31)
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    set_detail("cudaGetDevice failed");
    return FA2_ERR_CUDA;
  }
  if (dev >= 32 || !(attr_done_mask.load(std::memory_order_acquire) & (1u << dev))) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (e != cudaSuccess) {
      set_detail("cudaFuncSetAttribute: %s", cudaGetErrorString(e));
      return FA2_ERR_CUDA;
    }
    if (dev < 32) attr_done_mask.fetch_or(1u << dev, std::memory_order_acq_rel);
  }
  kern<<<dim3(n_q_tiles, prm.BH, splits), SKV_THREADS, C::SMEM_BYTES, stream>>>(tq, tk, tv, prm);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_detail("split-K/V kernel launch: %s", cudaGetErrorString(e));
    return FA2_ERR_CUDA;
  }
  if (prm.direct) return FA2_OK;
  const int rows = prm.BH * prm.Nq;
  fa2_splitkv_combine_kernel<HD><<<(rows + 3) / 4, 128, 0, stream>>>(prm.o_part, prm.lse_part, o, lse, rows, splits,
                                                                      prm.d);
  e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_detail("merge kernel launch: %s", cudaGetErrorString(e));
    return FA2_ERR_CUDA;
  }
  return FA2_OK;
}

static int splitkv_impl(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Nq,
                        int Nk, int d, int causal, float scale, int n_splits, void* workspace,
                        size_t workspace_bytes, unsigned long long timeout_ns, int inject, cudaStream_t stream) {
  g_detail[0] = 0;
  if (!q || !k || !v || !o || !lse) {
    set_detail("null pointer");
    return FA2_ERR_INVALID_ARG;
  }
  if (!skv_sizes_ok(B, H, Nq, Nk) || n_splits < 0) {
    set_detail("bad sizes B=%d H=%d Nq=%d Nk=%d n_splits=%d (need Nq >= 1, Nk >= Nq, B*H <= 65535)", B, H, Nq,
               Nk, n_splits);
    return FA2_ERR_INVALID_ARG;
  }
  if (!std::isfinite(scale) || !(scale > 0.f)) {
    set_detail("scale must be finite and positive");
    return FA2_ERR_INVALID_ARG;
  }
  if (!d_supported(d)) {
    set_detail("head dimension %d not supported (32, 64, 96, 128 or 256)", d);
    return FA2_ERR_UNSUPPORTED;
  }
  const uintptr_t mis = reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) |
                        reinterpret_cast<uintptr_t>(v) | reinterpret_cast<uintptr_t>(o);
  if ((mis & 15u) || (reinterpret_cast<uintptr_t>(lse) & 3u)) {
    set_detail("misaligned pointer (q/k/v/o need 16 bytes, lse 4)");
    return FA2_ERR_INVALID_ARG;
  }
  const int splits = skv_resolve_splits(B, H, Nq, Nk, n_splits, skv_tile_keys(d));
  const size_t need = skv_workspace_bytes(B, H, Nq, padded_hd(d), splits);
  if (need > 0 && (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || workspace_bytes < need)) {
    set_detail("workspace missing, misaligned or too small: %zu bytes, need %zu (256-byte aligned) for %d key ranges",
               workspace_bytes, need, splits);
    return FA2_ERR_INVALID_ARG;
  }
  const size_t BH = static_cast<size_t>(B) * H;
  const size_t qb = BH * Nq * d * 2, kb = BH * Nk * d * 2, lb = BH * Nq * 4;
  if (overlap(o, qb, q, qb) || overlap(o, qb, k, kb) || overlap(o, qb, v, kb) || overlap(o, qb, lse, lb) ||
      overlap(lse, lb, q, qb) || overlap(lse, lb, k, kb) || overlap(lse, lb, v, kb) ||
      (need > 0 && (overlap(workspace, need, q, qb) || overlap(workspace, need, k, kb) ||
                    overlap(workspace, need, v, kb) || overlap(workspace, need, o, qb) ||
                    overlap(workspace, need, lse, lb)))) {
    set_detail("output or workspace buffers overlap inputs or each other");
    return FA2_ERR_INVALID_ARG;
  }
  // Quarter mode for at most 32 query rows (d <= 128): 32-row query boxes.
  const bool quad = Nq <= 32 && padded_hd(d) <= 128;
  CUtensorMap tq, tk, tv;
  int st;
  if ((st = make_tmap(&tq, q, d, Nq, static_cast<int>(BH), quad ? 32 : 128)) != FA2_OK) return st;
  if ((st = make_tmap(&tk, k, d, Nk, static_cast<int>(BH), skv_tile_keys(d))) != FA2_OK) return st;
  if ((st = make_tmap(&tv, v, d, Nk, static_cast<int>(BH), skv_tile_keys(d))) != FA2_OK) return st;
  SkvParams prm;
  prm.direct = splits == 1;
  prm.o = static_cast<__nv_bfloat16*>(o);
  prm.lse = lse;
  prm.o_part = prm.direct ? nullptr : static_cast<float*>(workspace);
  prm.lse_part = prm.direct ? nullptr
                            : reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                                       round256(static_cast<size_t>(splits) * BH * Nq * padded_hd(d) * 4));
  prm.Nq = Nq;
  prm.Nk = Nk;
  prm.d = d;
  prm.BH = static_cast<int>(BH);
  prm.n_kv_tiles = (Nk + skv_tile_keys(d) - 1) / skv_tile_keys(d);
  prm.tiles_per_split = (prm.n_kv_tiles + splits - 1) / splits;
  prm.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634074);
  prm.timeout_ns = timeout_ns;
  prm.inject_timeout = inject;
  const int n_q_tiles = (Nq + BM - 1) / BM;
  auto* ob = static_cast<__nv_bfloat16*>(o);
  if (padded_hd(d) == 64) {
    if (quad)
      return causal ? skv_launch_t<64, true, true>(tq, tk, tv, prm, n_q_tiles, splits, ob, lse, stream)
                    : skv_launch_t<64, false, true>(tq, tk, tv, prm, n_q_tiles, splits, ob, lse, stream);
    return causal ? skv_launch_t<64, true, false>(tq, tk, tv, prm, n_q_tiles, splits, ob, lse, stream)
                  : skv_launch_t<64, false, false>(tq, tk, tv, prm, n_q_tiles, splits, ob, lse, stream);
  }
  if (padded_hd(d) == 256)
    return causal ? skv_launch_t<256, true, false>(tq, tk, tv, prm, n_q_tiles, splits, ob, lse, stream)
                  : skv_launch_t<256, false, false>(tq, tk, tv, prm, n_q_tiles, splits, ob, lse, stream);
  if (quad)
    return causal ? skv_launch_t<128, true, true>(tq, tk, tv, prm, n_q_tiles, splits, ob, lse, stream)
                  : skv_launch_t<128, false, true>(tq, tk, tv, prm, n_q_tiles, splits, ob, lse, stream);
  return causal ? skv_launch_t<128, true, false>(tq, tk, tv, prm, n_q_tiles, splits, ob, lse, stream)
                : skv_launch_t<128, false, false>(tq, tk, tv, prm, n_q_tiles, splits, ob, lse, stream);
}

// ------------------------------------------------------------------ backward host side

// Workspace of the backward: lse2 then D, fp32 [B*H, ceil(N/128)*128] each,
// each starting on a 256-byte boundary.
static size_t bwd_workspace_bytes_for(int B, int H, int N) {
  const size_t rows = static_cast<size_t>(B) * H * static_cast<size_t>((N + BM - 1) / BM) * BM;
  return 2 * round256(rows * 4);
}

template <typename Kern>
static int bwd_set_smem(Kern kern, int bytes) {
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) {
    set_detail("cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    return FA2_ERR_CUDA;
  }
  return FA2_OK;
}

// Maps: the dQ kernel reads 128-row Q and dO tiles and BNK-row K and V
// tiles; the dK/dV kernel 128-row K and V tiles and BMQ-row Q and dO tiles
// (the same maps when both are 128, i.e. d <= 128).
struct BwdMaps {
  CUtensorMap q128, do128, k_dq, v_dq;  // dQ kernel
  CUtensorMap k128, v128, q_kv, do_kv;  // dK/dV kernel(s)
  CUtensorMap dq128, dk128, dv128;       // gradient stores (128-row boxes)
};

template <int HD, bool CAUSAL>
static int bwd_launch_t(const BwdMaps& m, const BwdParams& prm, cudaStream_t stream) {
  using C = BwdCfg<HD>;
  static std::atomic<unsigned> attr_done_mask{0};  // per device bit (devices 0..31)
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    set_detail("cudaGetDevice failed");
    return FA2_ERR_CUDA;
  }
  constexpr int PASS0 = (HD == 256) ? BWD_KV_DV : BWD_KV_BOTH;
  auto kq = fa2_bwd_dq_kernel<HD, CAUSAL>;
  auto kkv = fa2_bwd_dkdv_kernel<HD, CAUSAL, PASS0>;
  if (dev >= 32 || !(attr_done_mask.load(std::memory_order_acquire) & (1u << dev))) {
    int st = bwd_set_smem(kq, C::DQ_SMEM);
    if (st == FA2_OK) st = bwd_set_smem(kkv, C::KV_SMEM);
    if constexpr (HD == 256)
      if (st == FA2_OK) st = bwd_set_smem(fa2_bwd_dkdv_kernel<HD, CAUSAL, BWD_KV_DK>, C::KV_SMEM);
    if (st != FA2_OK) return st;
    if (dev < 32) attr_done_mask.fetch_or(1u << dev, std::memory_order_acq_rel);
  }
  const unsigned grid = static_cast<unsigned>(prm.BH) * static_cast<unsigned>(prm.n_tiles);
  kq<<<grid, BWD_THREADS, C::DQ_SMEM, stream>>>(m.q128, m.k_dq, m.v_dq, m.do128, m.dq128, prm);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_detail("dQ kernel launch: %s", cudaGetErrorString(e));
    return FA2_ERR_CUDA;
  }
  kkv<<<grid, BWD_THREADS, C::KV_SMEM, stream>>>(m.q_kv, m.k128, m.v128, m.do_kv, m.dk128, m.dv128, prm);
  e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_detail("dK/dV kernel launch: %s", cudaGetErrorString(e));
    return FA2_ERR_CUDA;
  }
  if constexpr (HD == 256) {
    fa2_bwd_dkdv_kernel<HD, CAUSAL, BWD_KV_DK><<<grid, BWD_THREADS, C::KV_SMEM, stream>>>(
        m.q_kv, m.k128, m.v128, m.do_kv, m.dk128, m.dv128, prm);
    e = cudaGetLastError();
    if (e != cudaSuccess) {
      set_detail("dK kernel launch: %s", cudaGetErrorString(e));
      return FA2_ERR_CUDA;
    }
  }
  return FA2_OK;
}

static int bwd_impl(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
                    void* dq, void* dk, void* dv, int B, int H, int N, int d, int causal, float scale,
                    void* workspace, size_t workspace_bytes, unsigned long long timeout_ns, int inject,
                    cudaStream_t stream) {
  g_detail[0] = 0;
  if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv || !workspace) {
    set_detail("null pointer");
    return FA2_ERR_INVALID_ARG;
  }
  if (B < 1 || H < 1 || N < 1 || B > 65535 || H > 65535 ||
      static_cast<long long>(B) * H * ((N + BM - 1) / BM) > 0x7fffffffLL) {
    set_detail("bad sizes B=%d H=%d N=%d (need B, H <= 65535 and B*H*ceil(N/128) < 2^31)", B, H, N);
    return FA2_ERR_INVALID_ARG;
  }
  if (!std::isfinite(scale) || !(scale > 0.f)) {
    set_detail("scale must be finite and positive");
    return FA2_ERR_INVALID_ARG;
  }
  if (!d_supported(d)) {
    set_detail("head dimension %d not supported (32, 64, 96, 128 or 256)", d);
    return FA2_ERR_UNSUPPORTED;
  }
  const uintptr_t mis = reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) |
                        reinterpret_cast<uintptr_t>(v) | reinterpret_cast<uintptr_t>(o) |
                        reinterpret_cast<uintptr_t>(dout) | reinterpret_cast<uintptr_t>(dq) |
                        reinterpret_cast<uintptr_t>(dk) | reinterpret_cast<uintptr_t>(dv);
  if ((mis & 15u) || (reinterpret_cast<uintptr_t>(lse) & 3u) || (reinterpret_cast<uintptr_t>(workspace) & 255u)) {
    set_detail("misaligned pointer (tensors need 16 bytes, lse 4, workspace 256)");
    return FA2_ERR_INVALID_ARG;
  }
  const size_t need = bwd_workspace_bytes_for(B, H, N);
  if (workspace_bytes < need) {
    set_detail("workspace too small: %zu bytes, need %zu", workspace_bytes, need);
    return FA2_ERR_INVALID_ARG;
  }
  const size_t BH = static_cast<size_t>(B) * H;
  const size_t tb = BH * N * d * 2, lb = BH * N * 4;
  const void* ins[6] = {q, k, v, o, dout, lse};
  const size_t in_bytes[6] = {tb, tb, tb, tb, tb, lb};
  void* outs[4] = {dq, dk, dv, workspace};
  const size_t out_bytes[4] = {tb, tb, tb, need};
  for (int a = 0; a < 4; ++a) {
    for (int b = 0; b < 6; ++b)
      if (overlap(outs[a], out_bytes[a], ins[b], in_bytes[b])) {
        set_detail("output or workspace buffers overlap inputs");
        return FA2_ERR_INVALID_ARG;
      }
    for (int b = a + 1; b < 4; ++b)
      if (overlap(outs[a], out_bytes[a], outs[b], out_bytes[b])) {
        set_detail("output or workspace buffers overlap each other");
        return FA2_ERR_INVALID_ARG;
      }
  }
  // d = 256: 64-key tiles in the dQ kernel, 64-query tiles in the dK/dV kernels.
  const int tile_small = padded_hd(d) == 256 ? 64 : 128;
  BwdMaps maps;
  int st;
  const int bhi = static_cast<int>(BH);
  if ((st = make_tmap(&maps.q128, q, d, N, bhi)) != FA2_OK) return st;
  if ((st = make_tmap(&maps.do128, dout, d, N, bhi)) != FA2_OK) return st;
  if ((st = make_tmap(&maps.k128, k, d, N, bhi)) != FA2_OK) return st;
  if ((st = make_tmap(&maps.v128, v, d, N, bhi)) != FA2_OK) return st;
  if ((st = make_tmap(&maps.k_dq, k, d, N, bhi, tile_small)) != FA2_OK) return st;
  if ((st = make_tmap(&maps.v_dq, v, d, N, bhi, tile_small)) != FA2_OK) return st;
  if ((st = make_tmap(&maps.q_kv, q, d, N, bhi, tile_small)) != FA2_OK) return st;
  if ((st = make_tmap(&maps.do_kv, dout, d, N, bhi, tile_small)) != FA2_OK) return st;
  if ((st = make_tmap(&maps.dq128, dq, d, N, bhi)) != FA2_OK) return st;
  if ((st = make_tmap(&maps.dk128, dk, d, N, bhi)) != FA2_OK) return st;
  if ((st = make_tmap(&maps.dv128, dv, d, N, bhi)) != FA2_OK) return st;
  BwdParams prm;
  prm.o = static_cast<const __nv_bfloat16*>(o);
  prm.dout = static_cast<const __nv_bfloat16*>(dout);
  prm.lse = lse;
  prm.n_tiles = (N + BM - 1) / BM;
  prm.n_ktiles = (N + tile_small - 1) / tile_small;
  prm.n_qtiles = (N + tile_small - 1) / tile_small;
  prm.lse2 = static_cast<float*>(workspace);
  prm.dvec = reinterpret_cast<float*>(static_cast<char*>(workspace) + need / 2);
  prm.dq = static_cast<__nv_bfloat16*>(dq);
  prm.dk = static_cast<__nv_bfloat16*>(dk);
  prm.dv = static_cast<__nv_bfloat16*>(dv);
  prm.N = N;
  prm.d = d;
  prm.BH = static_cast<int>(BH);
  prm.group_heads = causal ? causal_group_heads(static_cast<int>(BH), N, d, prm.n_tiles) : 1;
  prm.scale = scale;
  prm.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634074);
  prm.timeout_ns = timeout_ns;
  prm.inject_timeout = inject;
  if (padded_hd(d) == 64)
    return causal ? bwd_launch_t<64, true>(maps, prm, stream) : bwd_launch_t<64, false>(maps, prm, stream);
  if (padded_hd(d) == 256)
    return causal ? bwd_launch_t<256, true>(maps, prm, stream) : bwd_launch_t<256, false>(maps, prm, stream);
  return causal ? bwd_launch_t<128, true>(maps, prm, stream) : bwd_launch_t<128, false>(maps, prm, stream);
}

// ------------------------------------------------------------------ split-K/V with library-owned scratch
// For callers that cannot allocate device memory (see fa2_fwd_splitkv_static
// in fa2.h): the partial outputs live in this fixed array instead of a
// caller workspace.  Every device that loads the library holds it until the
// process exits.  Nothing in it has to start at zero: each call writes every
// partial the merge reads.  All calls share it, so calls that overlap on the
// GPU (other streams, other host threads) race on its contents.
static __device__ __align__(256) unsigned char g_skv_static_scratch[FA2_SPLITKV_STATIC_SCRATCH_BYTES];

constexpr int MAX_DEVICES = 64;
static std::mutex g_static_scratch_mu;
static void* g_static_scratch_addr[MAX_DEVICES] = {};

// Device address of the scratch array on the current device.  The host-side
// name g_skv_static_scratch is only a stand-in for the symbol; the address is
// looked up once per device (the first call on that device) and cached.
static int static_scratch_on_current_device(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    set_detail("cudaGetDevice: %s", cudaGetErrorString(e));
    return FA2_ERR_CUDA;
  }
  if (dev < 0 || dev >= MAX_DEVICES) {
    set_detail("device %d is beyond the %d devices the static scratch table covers", dev, MAX_DEVICES);
    return FA2_ERR_UNSUPPORTED;
  }
  std::lock_guard<std::mutex> lock(g_static_scratch_mu);
  if (!g_static_scratch_addr[dev]) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_skv_static_scratch);
    if (e != cudaSuccess || !ptr) {
      set_detail("cudaGetSymbolAddress of the static scratch: %s", cudaGetErrorString(e));
      return FA2_ERR_CUDA;
    }
    g_static_scratch_addr[dev] = ptr;
  }
  *out = g_static_scratch_addr[dev];
  return FA2_OK;
}

}  // namespace fa2

// ====================================================================== C ABI
extern "C" {

int fa2_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d,
            int causal, float scale, void* stream) {
  return fa2::fwd_impl(q, k, v, o, lse, B, H, N, d, causal, scale, fa2::DEFAULT_TIMEOUT_NS, 0,
                       static_cast<cudaStream_t>(stream));
}

int fa2_fwd_inject_timeout(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                           int N, int d, int causal, float scale, unsigned long long timeout_ns, void* stream) {
  if (timeout_ns == 0 || timeout_ns > fa2::DEFAULT_TIMEOUT_NS) {
    fa2::set_detail("timeout_ns out of range (1 .. 2e9)");
    return FA2_ERR_INVALID_ARG;
  }
  return fa2::fwd_impl(q, k, v, o, lse, B, H, N, d, causal, scale, timeout_ns, 1,
                       static_cast<cudaStream_t>(stream));
}

int fa2_sync_status(void* stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) {
    fa2::set_detail("cudaStreamSynchronize: %s", cudaGetErrorString(e));
    return FA2_ERR_CUDA;
  }
  unsigned int st = 0;
  e = cudaMemcpyFromSymbol(&st, fa2::g_fa2_status, sizeof(st));
  if (e != cudaSuccess) {
    fa2::set_detail("reading the status word: %s", cudaGetErrorString(e));
    return FA2_ERR_CUDA;
  }
  if (st) {
    const unsigned int zero = 0;
    cudaMemcpyToSymbol(fa2::g_fa2_status, &zero, sizeof(zero));
    fa2::set_detail("device status word 0x%x", st);
    return FA2_ERR_TIMEOUT;
  }
  return FA2_OK;
}

size_t fa2_fwd_host_workspace_bytes(int B, int H, int N, int d) {
  if (B < 1 || H < 1 || N < 1 || !fa2::d_supported(d)) return 0;
  const size_t t = ((static_cast<size_t>(B) * H * N * d * 2) + 255) & ~static_cast<size_t>(255);
  const size_t l = ((static_cast<size_t>(B) * H * N * 4) + 255) & ~static_cast<size_t>(255);
  return 4 * t + l;
}

int fa2_fwd_host(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d,
                 int causal, float scale, void* workspace, size_t workspace_bytes, void* stream) {
  fa2::g_detail[0] = 0;
  if (!q || !k || !v || !o || !lse || !workspace) {
    fa2::set_detail("null pointer");
    return FA2_ERR_INVALID_ARG;
  }
  const size_t need = fa2_fwd_host_workspace_bytes(B, H, N, d);
  if (need == 0) {
    if (!fa2::d_supported(d) && B >= 1 && H >= 1 && N >= 1) return FA2_ERR_UNSUPPORTED;
    fa2::set_detail("bad sizes");
    return FA2_ERR_INVALID_ARG;
  }
  if (workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u)) {
    fa2::set_detail("workspace too small or misaligned (need %zu bytes, 256-byte aligned)", need);
    return FA2_ERR_INVALID_ARG;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t tb = static_cast<size_t>(B) * H * N * d * 2;
  const size_t t = (tb + 255) & ~static_cast<size_t>(255);
  char* ws = static_cast<char*>(workspace);
  char *dq = ws, *dk = ws + t, *dv = ws + 2 * t, *dout = ws + 3 * t;
  float* dl = reinterpret_cast<float*>(ws + 4 * t);
  // Validate once on the whole shape before any copy is queued.
  {
    const int st = fa2::validate(dq, dk, dv, dout, dl, B, H, N, d, scale);
    if (st != FA2_OK) return st;
  }
  fa2::HostPipe* pipe = nullptr;
  {
    const int st = fa2::host_pipe(&pipe);
    if (st != FA2_OK) return st;
  }
  std::lock_guard<std::mutex> lock(pipe->mu);
  // The B*H heads are contiguous ([B, H, N, d]), so a run of heads is one
  // contiguous slice of every tensor.  Chunk c is uploaded on the caller's
  // stream, computed on the pipe's compute stream once its upload is done, and
  // downloaded on the pipe's download stream once computed: the copies of
  // neighbouring chunks overlap each other (both copy directions) and the
  // kernels.  Every head is computed exactly as in one whole call.
  // Chunks are runs of whole batches when there are enough batches (each
  // chunk then keeps the caller's H), else runs of heads (each shorter than H).
  const long long BH = static_cast<long long>(B) * H;
  const int chunks = static_cast<int>(std::min<long long>(fa2::HostPipe::MAX_CHUNKS, BH));
  const bool by_batch = B >= chunks;
  const size_t head_b = static_cast<size_t>(N) * d * 2, head_l = static_cast<size_t>(N) * 4;
  cudaError_t e = cudaSuccess;
  int st = FA2_OK;
  int c = 0;
  for (; c < chunks; ++c) {
    const long long u0 = (by_batch ? B : BH) * c / chunks, u1 = (by_batch ? B : BH) * (c + 1) / chunks;
    const long long h0 = by_batch ? u0 * H : u0, h1 = by_batch ? u1 * H : u1;
    const int cB = by_batch ? static_cast<int>(u1 - u0) : 1, cH = by_batch ? H : static_cast<int>(u1 - u0);
    const size_t ob = static_cast<size_t>(h0) * head_b, nb = static_cast<size_t>(h1 - h0) * head_b;
    const size_t ol = static_cast<size_t>(h0) * head_l, nl = static_cast<size_t>(h1 - h0) * head_l;
    if ((e = cudaMemcpyAsync(dq + ob, static_cast<const char*>(q) + ob, nb, cudaMemcpyHostToDevice, s)) != cudaSuccess ||
        (e = cudaMemcpyAsync(dk + ob, static_cast<const char*>(k) + ob, nb, cudaMemcpyHostToDevice, s)) != cudaSuccess ||
        (e = cudaMemcpyAsync(dv + ob, static_cast<const char*>(v) + ob, nb, cudaMemcpyHostToDevice, s)) != cudaSuccess ||
        (e = cudaEventRecord(pipe->uploaded[c], s)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(pipe->compute, pipe->uploaded[c], 0)) != cudaSuccess) {
      fa2::set_detail("host-to-device copy: %s", cudaGetErrorString(e));
      st = FA2_ERR_CUDA;
      break;
    }
    st = fa2_fwd(dq + ob, dk + ob, dv + ob, dout + ob, dl + h0 * N, cB, cH, N, d, causal, scale, pipe->compute);
    if (st != FA2_OK) break;
    if ((e = cudaEventRecord(pipe->computed[c], pipe->compute)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(pipe->download, pipe->computed[c], 0)) != cudaSuccess ||
        (e = cudaMemcpyAsync(static_cast<char*>(o) + ob, dout + ob, nb, cudaMemcpyDeviceToHost, pipe->download)) !=
            cudaSuccess ||
        (e = cudaMemcpyAsync(reinterpret_cast<char*>(lse) + ol, reinterpret_cast<char*>(dl) + ol, nl,
                             cudaMemcpyDeviceToHost, pipe->download)) != cudaSuccess) {
      fa2::set_detail("device-to-host copy: %s", cudaGetErrorString(e));
      st = FA2_ERR_CUDA;
      break;
    }
  }
  // The caller's stream is ordered after everything queued on the pipe's
  // streams (also on an error part-way), so its synchronisation covers them.
  if ((e = cudaEventRecord(pipe->drained, pipe->download)) != cudaSuccess ||
      (e = cudaStreamWaitEvent(s, pipe->drained, 0)) != cudaSuccess ||
      (e = cudaEventRecord(pipe->drained, pipe->compute)) != cudaSuccess ||
      (e = cudaStreamWaitEvent(s, pipe->drained, 0)) != cudaSuccess) {
    cudaStreamSynchronize(pipe->compute);
    cudaStreamSynchronize(pipe->download);
    if (st == FA2_OK) {
      fa2::set_detail("stream ordering: %s", cudaGetErrorString(e));
      st = FA2_ERR_CUDA;
    }
  }
  if (st != FA2_OK) {
    cudaStreamSynchronize(s);
    return st;
  }
  return fa2_sync_status(stream);
}

int fa2_fwd_splitkv_splits(int B, int H, int Nq, int Nk, int d, int n_splits) {
  if (!fa2::skv_sizes_ok(B, H, Nq, Nk) || n_splits < 0 || !fa2::d_supported(d)) return 0;
  return fa2::skv_resolve_splits(B, H, Nq, Nk, n_splits, fa2::skv_tile_keys(d));
}

size_t fa2_fwd_splitkv_workspace_bytes(int B, int H, int Nq, int Nk, int d, int n_splits) {
  const int splits = fa2_fwd_splitkv_splits(B, H, Nq, Nk, d, n_splits);
  if (splits == 0) return 0;
  return fa2::skv_workspace_bytes(B, H, Nq, fa2::padded_hd(d), splits);
}

int fa2_fwd_splitkv(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Nq, int Nk,
                    int d, int causal, float scale, int n_splits, void* workspace, size_t workspace_bytes,
                    void* stream) {
  return fa2::splitkv_impl(q, k, v, o, lse, B, H, Nq, Nk, d, causal, scale, n_splits, workspace, workspace_bytes,
                           fa2::DEFAULT_TIMEOUT_NS, 0, static_cast<cudaStream_t>(stream));
}

int fa2_fwd_splitkv_inject_timeout(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                                   int Nq, int Nk, int d, int causal, float scale, int n_splits, void* workspace,
                                   size_t workspace_bytes, unsigned long long timeout_ns, void* stream) {
  if (timeout_ns == 0 || timeout_ns > fa2::DEFAULT_TIMEOUT_NS) {
    fa2::set_detail("timeout_ns out of range (1 .. 2e9)");
    return FA2_ERR_INVALID_ARG;
  }
  return fa2::splitkv_impl(q, k, v, o, lse, B, H, Nq, Nk, d, causal, scale, n_splits, workspace, workspace_bytes,
                           timeout_ns, 1, static_cast<cudaStream_t>(stream));
}

int fa2_fwd_splitkv_static(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Nq,
                           int Nk, int d, int causal, float scale, int n_splits, void* stream) {
  fa2::g_detail[0] = 0;
  if (!q || !k || !v || !o || !lse) {
    fa2::set_detail("null pointer");
    return FA2_ERR_INVALID_ARG;
  }
  size_t need = 0;
  if (fa2::skv_sizes_ok(B, H, Nq, Nk) && n_splits >= 0 && fa2::d_supported(d)) {
    const int splits = fa2::skv_resolve_splits(B, H, Nq, Nk, n_splits, fa2::skv_tile_keys(d));
    need = fa2::skv_workspace_bytes(B, H, Nq, fa2::padded_hd(d), splits);
    if (need > FA2_SPLITKV_STATIC_SCRATCH_BYTES) {
      fa2::set_detail("%d key ranges need %zu bytes of scratch; the static scratch holds %zu (fewer ranges need "
                      "less, one range none; fa2_fwd_splitkv takes a caller workspace of any size)",
                      splits, need, static_cast<size_t>(FA2_SPLITKV_STATIC_SCRATCH_BYTES));
      return FA2_ERR_INVALID_ARG;
    }
  }
  void* scratch = nullptr;
  if (need > 0) {
    const int st = fa2::static_scratch_on_current_device(&scratch);
    if (st != FA2_OK) return st;
  }
  return fa2::splitkv_impl(q, k, v, o, lse, B, H, Nq, Nk, d, causal, scale, n_splits, scratch,
                           scratch ? static_cast<size_t>(FA2_SPLITKV_STATIC_SCRATCH_BYTES) : 0,
                           fa2::DEFAULT_TIMEOUT_NS, 0, static_cast<cudaStream_t>(stream));
}

size_t fa2_bwd_workspace_bytes(int B, int H, int N, int d) {
  if (B < 1 || H < 1 || N < 1 || !fa2::d_supported(d)) return 0;
  return fa2::bwd_workspace_bytes_for(B, H, N);
}

int fa2_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse, void* dq,
            void* dk, void* dv, int B, int H, int N, int d, int causal, float scale, void* workspace,
            size_t workspace_bytes, void* stream) {
  return fa2::bwd_impl(q, k, v, o, dout, lse, dq, dk, dv, B, H, N, d, causal, scale, workspace, workspace_bytes,
                       fa2::DEFAULT_TIMEOUT_NS, 0, static_cast<cudaStream_t>(stream));
}

int fa2_bwd_inject_timeout(const void* q, const void* k, const void* v, const void* o, const void* dout,
                           const float* lse, void* dq, void* dk, void* dv, int B, int H, int N, int d, int causal,
                           float scale, void* workspace, size_t workspace_bytes, int kernel,
                           unsigned long long timeout_ns, void* stream) {
  if (timeout_ns == 0 || timeout_ns > fa2::DEFAULT_TIMEOUT_NS) {
    fa2::set_detail("timeout_ns out of range (1 .. 2e9)");
    return FA2_ERR_INVALID_ARG;
  }
  if (kernel != 0 && kernel != 1) {
    fa2::set_detail("kernel must be 0 (dQ) or 1 (dK/dV)");
    return FA2_ERR_INVALID_ARG;
  }
  return fa2::bwd_impl(q, k, v, o, dout, lse, dq, dk, dv, B, H, N, d, causal, scale, workspace, workspace_bytes,
                       timeout_ns, kernel + 1, static_cast<cudaStream_t>(stream));
}

const char* fa2_strerror(int status) {
  switch (status) {
    case FA2_OK: return "ok";
    case FA2_ERR_INVALID_ARG: return "invalid argument";
    case FA2_ERR_UNSUPPORTED: return "unsupported configuration";
    case FA2_ERR_CUDA: return "CUDA error";
    case FA2_ERR_TIMEOUT: return "kernel wait timed out";
    default: return "unknown status";
  }
}

const char* fa2_last_error_detail(void) { return fa2::g_detail; }

int fa2_version(void) { return 100; }

#ifdef FA2_TRACE
// Trace builds only: copy the timeline ((32 events x 64 tiles) + start) to host.
int fa2_trace_read(long long* host, int n) {
  if (!host || n < fa2::TRACE_EV * fa2::TRACE_J + 1) return FA2_ERR_INVALID_ARG;
  return cudaMemcpyFromSymbol(host, fa2::g_fa2_trace, sizeof(long long) * (fa2::TRACE_EV * fa2::TRACE_J + 1)) ==
                 cudaSuccess
             ? FA2_OK
             : FA2_ERR_CUDA;
}
#endif

}  // extern "C"
