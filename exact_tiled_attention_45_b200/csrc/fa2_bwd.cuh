// Backward pass of exact attention.  Included by fa2_fwd.cu inside
// namespace fa2 (one translation unit: shares the status word and helpers).
//
// Given Q, K, V, the forward output O, its per-row logsumexp LSE and the
// upstream gradient dO, with P = exp(scale * Q K^T - LSE) (masked entries 0):
//     D_i = sum_k dO_ik O_ik          (= sum_j P_ij dP_ij, since O = P V)
//     dV  = P^T dO
//     dP  = dO V^T
//     dS  = P o (dP - D)              (o: elementwise; D broadcast along rows)
//     dQ  = scale * dS K
//     dK  = scale * dS^T Q
// The pages state only that gradients are compared with tolerances (iplexlaw
// blog "FlashAttention-2: making long-context attention run efficiently on
// GPUs", section "Tiling preserves the attention calculation"); the formulas
// are the chain rule through the forward definition, and the forward LSE is
// what lets P be recomputed tile by tile without a second softmax pass.
//
// Two kernels, no atomics.  Each keeps one 128-row tile resident and streams
// the other operand's tiles, with P and dS recomputed per tile pair:
//   fa2_bwd_dq_kernel    one CTA per query tile: S = Q K_j^T, dP = dO V_j^T,
//                        dQ += dS K_j (3 MMAs per key tile); it also writes
//                        -LSE * log2(e) and D per row to the workspace;
//   fa2_bwd_dkdv_kernel  one CTA per key tile: S^T = K Q_i^T, dP^T = V dO_i^T,
//                        dV += P^T dO_i, dK += dS^T Q_i (4 MMAs per query tile).
// Seven MMAs per tile pair instead of five: dQ is not accumulated across CTAs.
//
// Roles (192 threads): warps 0-3 elementwise (thread r <-> tile row r <->
// TMEM lane r), warp 4 TMA producer, warp 5 MMA issuer.  P (dK/dV kernel) and
// dS are packed to bf16 over the first half of their score tile's columns in
// TMEM and read from there by the next MMA.  Every wait is bounded.
//
// Head dimension 256: the dQ kernel streams 64-key tiles (TMEM: S 64, dP 64
// and a 256-column dQ; shared memory: Q and dO 128 KB, two K stages, one V
// stage), and the dK/dV kernel runs twice over 64-query tiles, once for dV
// (S^T, dV += P^T dO: 320 TMEM columns) and once for dK (S^T, dP^T,
// dK += dS^T Q: 384 columns), since S^T, dP^T, dV and dK together would need
// 768 of the 512 columns.  Eight MMAs per tile pair.

constexpr int BWD_THREADS = 192;
constexpr int BWD_PRODUCER_WARP = 4;
constexpr int BWD_MMA_WARP = 5;
constexpr float LOG2E_F = 1.4426950408889634f;
// Of every 8 pairs of exponentials 2^(c*s - LSE*log2(e)), this many run on
// the FMA-pipe polynomial (exp2_poly_pair) and the rest on the
// special-function unit; the arguments are <= 0 (P <= 1), -inf when masked.
// Measured: 1 of 8 is fastest at d = 128 (+1.1 % over 2 at the headline
// shape), 2 of 8 at d = 64 (where the MMAs per exponential are half).
#ifndef FA2_BWD_EMU_PAIRS_D64
#define FA2_BWD_EMU_PAIRS_D64 2
#endif
#ifndef FA2_BWD_EMU_PAIRS_WIDE
#define FA2_BWD_EMU_PAIRS_WIDE 1  // d = 128 and 256
#endif

// P of NC keys (or queries) of one row: pr[e] = 2^(c * s[e] + nl[e]), where
// nl is -LSE*log2(e) (one value per row, or per column when `per_col`);
// masked entries (e past `lim` on a masked tile, see the callers) give 0.
template <bool PER_COL, int NC, int EMU>
__device__ __forceinline__ void bwd_probs(float (&pr)[NC], const uint32_t (&s)[NC], float c, float nl_row,
                                          const float* nl_col, bool masked, int lim, bool mask_below) {
  const uint64_t cc = f2_pack(c, c);
  const uint64_t nlr = f2_pack(nl_row, nl_row);
#pragma unroll
  for (int e = 0; e < NC; e += 2) {
    float x0 = __uint_as_float(s[e]), x1 = __uint_as_float(s[e + 1]);
    if (masked) {
      // mask_below: entries before `lim` are masked, else entries after it
      if (mask_below ? (e < lim) : (e > lim)) x0 = -INFINITY;
      if (mask_below ? (e + 1 < lim) : (e + 1 > lim)) x1 = -INFINITY;
    }
    uint64_t nl = nlr;
    if (PER_COL) nl = *reinterpret_cast<const uint64_t*>(nl_col + e);
    const uint64_t x = f2_fma(f2_pack(x0, x1), cc, nl);
    if (((e >> 1) & 7) < EMU) {
      f2_unpack(exp2_poly_pair(x), pr[e], pr[e + 1]);
    } else {
      float a0, a1;
      f2_unpack(x, a0, a1);
      pr[e] = ex2(a0);
      pr[e + 1] = ex2(a1);
    }
  }
}

template <int HD>
struct BwdCfg {
  static_assert(HD == 64 || HD == 128 || HD == 256, "head dimension");
  static constexpr int KCH = HD / 64;
  static constexpr int EMU_PAIRS = (HD == 64) ? FA2_BWD_EMU_PAIRS_D64 : FA2_BWD_EMU_PAIRS_WIDE;
  static constexpr int CHUNK_BYTES = 128 * 128;          // 128 rows x 128 bytes
  static constexpr int TILE_BYTES = KCH * CHUNK_BYTES;   // one 128-row tile
  // dQ kernel: Q and dO resident, K and V rings of BNK-key tiles.
  static constexpr int BNK = (HD == 256) ? 64 : 128;
  static constexpr int KV_CHUNK = BNK * 128;
  static constexpr int KV_TILE = KCH * KV_CHUNK;
  static constexpr int DQ_KS = (HD == 256) ? 2 : (HD == 128 ? 3 : 4);
  static constexpr int DQ_VS = (HD == 256) ? 1 : (HD == 128 ? 2 : 4);
  static constexpr int DQ_OFF_Q = 0;
  static constexpr int DQ_OFF_DO = DQ_OFF_Q + TILE_BYTES;
  static constexpr int DQ_OFF_K = DQ_OFF_DO + TILE_BYTES;
  static constexpr int DQ_OFF_V = DQ_OFF_K + DQ_KS * KV_TILE;
  static constexpr int DQ_OFF_BAR = DQ_OFF_V + DQ_VS * KV_TILE;
  static constexpr int DQ_SMEM = DQ_OFF_BAR + 256 + 1024;
  // dK/dV kernel: K and V resident (128 keys), a ring of (Q_i, dO_i, lse2_i,
  // D_i) of BMQ-query tiles.
  static constexpr int BMQ = (HD == 256) ? 64 : 128;
  static constexpr int Q_CHUNK = BMQ * 128;
  static constexpr int Q_TILE = KCH * Q_CHUNK;
  static constexpr int KV_QS = (HD == 256) ? 1 : (HD == 128 ? 2 : 3);
  static constexpr int KV_OFF_K = 0;
  static constexpr int KV_OFF_V = TILE_BYTES;
  static constexpr int KV_OFF_Q = 2 * TILE_BYTES;
  static constexpr int KV_OFF_DO = KV_OFF_Q + KV_QS * Q_TILE;
  static constexpr int KV_OFF_VEC = KV_OFF_DO + KV_QS * Q_TILE;  // per stage: lse2[BMQ] at +0, D[BMQ] at +512
  static constexpr int KV_OFF_BAR = KV_OFF_VEC + KV_QS * 1024;
  static constexpr int KV_SMEM = KV_OFF_BAR + 256 + 1024;
  static_assert(DQ_SMEM <= 232448 && KV_SMEM <= 232448, "shared memory budget");
  static_assert(DQ_KS <= 4 && DQ_VS <= 4 && KV_QS <= 3, "barrier arrays");
};

// Passes of the dK/dV kernel: both gradients (d <= 128), or dV and dK in
// two launches (d = 256).
constexpr int BWD_KV_BOTH = 0, BWD_KV_DV = 1, BWD_KV_DK = 2;

struct BwdParams {
  const __nv_bfloat16* o;     // forward output [B*H, N, d]
  const __nv_bfloat16* dout;  // upstream gradient [B*H, N, d]
  const float* lse;           // forward logsumexp (natural log) [B*H, N]
  float* lse2;                // workspace [B*H, n_tiles*128]: -LSE * log2(e); -inf past N
  float* dvec;                // workspace [B*H, n_tiles*128]: D; 0 past N
  __nv_bfloat16* dq;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  int N;
  int d;            // head dimension of the tensors (<= HD; the kernel's tiles are zero-padded to HD)
  int BH;
  int n_tiles;      // ceil(N / 128): the dQ kernel's query tiles and the dK/dV kernel's key tiles
  int n_ktiles;     // ceil(N / BNK): key tiles streamed by the dQ kernel
  int n_qtiles;     // ceil(N / BMQ): query tiles streamed by the dK/dV kernel
  int group_heads;  // heads per launch-order group
  float scale;
  float scale_log2;
  unsigned long long timeout_ns;
  // Test hook: 1 withholds the dQ kernel's Q/dO load, 2 the dK/dV kernel's
  // K/V load, so that kernel's waits on it run out.
  int inject_timeout;
};

// Work item of a 1-D grid: heads in groups of group_heads, tile rank the slow
// index inside a group; with causal masking rank 0 is the heaviest tile (the
// last query tile for dQ, the first key tile for dK/dV).
template <bool CAUSAL, bool HEAVY_IS_LAST>
__device__ __forceinline__ void bwd_item(const BwdParams& p, int& bh, int& tile) {
  const int per_group = p.group_heads * p.n_tiles;
  const int grp = static_cast<int>(blockIdx.x) / per_group;
  const int in_grp = static_cast<int>(blockIdx.x) - grp * per_group;
  const int grp_heads = min(p.group_heads, p.BH - grp * p.group_heads);
  const int rank = in_grp / grp_heads;
  bh = grp * p.group_heads + (in_grp - rank * grp_heads);
  tile = (CAUSAL && HEAVY_IS_LAST) ? (p.n_tiles - 1 - rank) : rank;
}

// Row r of an NC-column fp32 accumulator in TMEM, times f, as bf16 into a
// 128-row tile in shared memory laid out for TMA stores of 64-column boxes
// with 128-byte swizzle: 64-column chunk c at tile + c * 16 KB, row r at
// r * 128 bytes, 16-byte unit k of the row at (k ^ (r mod 8)) * 16.  Up to
// 128 columns are loaded from TMEM at a time.
template <int NC>
__device__ __forceinline__ void stage_row_bf16(uint32_t tile, uint32_t taddr, int r, float f) {
  constexpr int G = (NC < 128 ? NC : 128) / 32;
  const uint64_t ff = f2_pack(f, f);
#pragma unroll
  for (int g = 0; g < NC / 32; g += G) {
    uint32_t a[G][32];
#pragma unroll
    for (int cc = 0; cc < G; ++cc) tmem_ld32(taddr + (g + cc) * 32, a[cc]);
    tmem_wait_ld();
#pragma unroll
    for (int cc = 0; cc < G; ++cc) reg_fence32(a[cc]);
#pragma unroll
    for (int cc = 0; cc < G; ++cc) {
      const int c32 = g + cc;
      uint32_t w[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        float x0, x1;
        f2_unpack(f2_mul(f2_pack(__uint_as_float(a[cc][2 * e]), __uint_as_float(a[cc][2 * e + 1])), ff), x0, x1);
        w[e] = pack_bf16x2(x0, x1);
      }
      const uint32_t line = tile + static_cast<uint32_t>(c32 >> 1) * (128u * 128u) + static_cast<uint32_t>(r) * 128u;
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const int k = (c32 & 1) * 4 + v;
        st_shared_v4(line + ((k ^ (r & 7)) << 4), w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
      }
    }
  }
}

// dS for NC keys (or queries) of one row: reads dP from TMEM 32 columns at a
// time and writes dS (bf16 pairs) over the first NC/2 columns.  Chunk q
// writes packed columns [16q, 16q+16), which held dP of keys 16q..16q+15:
// chunk q/2 <= q has already read them.
template <int NC>
__device__ __forceinline__ void ds_to_tmem(uint32_t dp_addr, const float (&p)[NC], const float* dsub, bool per_col,
                                           float dsub_row) {
#pragma unroll
  for (int q = 0; q < NC / 32; ++q) {
    uint32_t dp[32];
    tmem_ld32(dp_addr + 32 * q, dp);
    tmem_wait_ld();
    reg_fence32(dp);
    uint32_t pk[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const int c0 = 32 * q + 2 * e;
      const float d0 = per_col ? dsub[c0] : dsub_row;
      const float d1 = per_col ? dsub[c0 + 1] : dsub_row;
      pk[e] = pack_bf16x2(p[c0] * (__uint_as_float(dp[2 * e]) - d0), p[c0 + 1] * (__uint_as_float(dp[2 * e + 1]) - d1));
    }
    tmem_st16(dp_addr + 16 * q, pk);
  }
}

struct DqBars {
  uint64_t q_full, do_full;  // the resident Q and dO tiles (S waits for Q only)
  uint64_t k_full[4], k_empty[4];
  uint64_t v_full[4], v_empty[4];
  uint64_t s_full, s_free, dp_full, ds_ready, mma_final;
  uint64_t epi;  // the four elementwise warps staged their gradient rows in shared memory
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(DqBars) <= 256, "barrier block");

// TMEM columns of the dQ kernel: S [0,BNK), dP [128,128+BNK), dQ [256, 256+d).
constexpr uint32_t BQ_S = 0, BQ_DP = 128, BQ_DQ = 256;

template <int HD, bool CAUSAL>
__global__ void __launch_bounds__(BWD_THREADS, 1)
    fa2_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                      const __grid_constant__ CUtensorMap tm_dq, const BwdParams p) {
  using C = BwdCfg<HD>;
  constexpr int BNK = C::BNK;
  int bh, qt;
  bwd_item<CAUSAL, true>(p, bh, qt);
  const int q0 = qt * BM;
  // Key tiles up to the one holding this query tile's last row (causal).
  const int nkv = CAUSAL ? min((q0 + BM - 1) / BNK + 1, p.n_ktiles) : p.n_ktiles;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t base = (raw_addr + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw_addr);
  DqBars* bars = reinterpret_cast<DqBars*>(smem + C::DQ_OFF_BAR);
  volatile int* abort_flag = &bars->abort;
  const uint32_t sQ = base + C::DQ_OFF_Q, sDO = base + C::DQ_OFF_DO;
  const uint32_t sK = base + C::DQ_OFF_K, sV = base + C::DQ_OFF_V;

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bars->q_full), 1);
    mbar_init(smem_u32(&bars->do_full), 1);
    for (int s = 0; s < C::DQ_KS; ++s) {
      mbar_init(smem_u32(&bars->k_full[s]), 1);
      mbar_init(smem_u32(&bars->k_empty[s]), 1);
    }
    for (int s = 0; s < C::DQ_VS; ++s) {
      mbar_init(smem_u32(&bars->v_full[s]), 1);
      mbar_init(smem_u32(&bars->v_empty[s]), 1);
    }
    mbar_init(smem_u32(&bars->s_full), 1);
    mbar_init(smem_u32(&bars->s_free), 4);
    mbar_init(smem_u32(&bars->dp_full), 1);
    mbar_init(smem_u32(&bars->ds_ready), 4);
    mbar_init(smem_u32(&bars->mma_final), 1);
    mbar_init(smem_u32(&bars->epi), 4);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == BWD_MMA_WARP) {
    tmem_alloc(smem_u32(&bars->tmem_base), TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == BWD_PRODUCER_WARP && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    prefetch_tmap(&tm_do);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const unsigned long long to = p.timeout_ns;

  if (warp == BWD_PRODUCER_WARP) {
    if (lane == 0) {
      // Q, K(0), dO, V(0): the order the first two MMAs need them.
      const uint32_t bq = smem_u32(&bars->q_full), bdo = smem_u32(&bars->do_full);
      const bool load_qdo = p.inject_timeout != 1;
      if (load_qdo) {
        mbar_arrive_expect_tx(bq, C::TILE_BYTES);
        for (int c = 0; c < C::KCH; ++c) tma_load_3d(sQ + c * C::CHUNK_BYTES, &tm_q, bq, c * 64, q0, bh);
      }
      int k_issued = 0, v_issued = 0;
      for (int j = 0; j < nkv; ++j) {
        const int ks = j % C::DQ_KS, vs = j % C::DQ_VS;
        if (j >= C::DQ_KS &&
            !wait_bounded(smem_u32(&bars->k_empty[ks]), ((j / C::DQ_KS) - 1) & 1, abort_flag, to, ROLE_PRODUCER))
          break;
        const uint32_t kb = smem_u32(&bars->k_full[ks]);
        mbar_arrive_expect_tx(kb, C::KV_TILE);
        for (int c = 0; c < C::KCH; ++c)
          tma_load_3d(sK + ks * C::KV_TILE + c * C::KV_CHUNK, &tm_k, kb, c * 64, j * BNK, bh);
        ++k_issued;
        if (j == 0 && load_qdo) {
          mbar_arrive_expect_tx(bdo, C::TILE_BYTES);
          for (int c = 0; c < C::KCH; ++c) tma_load_3d(sDO + c * C::CHUNK_BYTES, &tm_do, bdo, c * 64, q0, bh);
        }
        if (j >= C::DQ_VS &&
            !wait_bounded(smem_u32(&bars->v_empty[vs]), ((j / C::DQ_VS) - 1) & 1, abort_flag, to, ROLE_PRODUCER))
          break;
        const uint32_t vb = smem_u32(&bars->v_full[vs]);
        mbar_arrive_expect_tx(vb, C::KV_TILE);
        for (int c = 0; c < C::KCH; ++c)
          tma_load_3d(sV + vs * C::KV_TILE + c * C::KV_CHUNK, &tm_v, vb, c * 64, j * BNK, bh);
        ++v_issued;
      }
      if (load_qdo) {
        wait_drain(bq, 0, to);
        if (k_issued > 0) wait_drain(bdo, 0, to);
      }
      for (int x = (k_issued > C::DQ_KS ? k_issued - C::DQ_KS : 0); x < k_issued; ++x)
        wait_drain(smem_u32(&bars->k_full[x % C::DQ_KS]), (x / C::DQ_KS) & 1, to);
      for (int x = (v_issued > C::DQ_VS ? v_issued - C::DQ_VS : 0); x < v_issued; ++x)
        wait_drain(smem_u32(&bars->v_full[x % C::DQ_VS]), (x / C::DQ_VS) & 1, to);
    }
  } else if (warp == BWD_MMA_WARP) {
    // S(0), dP(0); then per j >= 1: S(j), dQ(j-1), dP(j).  dS(j-1) lives in
    // dP's columns, so dP(j) is issued after dQ(j-1) has been (in order).
    if (lane == 0) {
      constexpr uint32_t IDESC_SS = idesc_bf16_f32(BM, BNK, false, false);
      constexpr uint32_t IDESC_DQ = idesc_bf16_f32(BM, HD, false, true);
      // A: a 128-row tile (Q or dO); B: a BNK-row tile (K or V); both K-major.
      auto mma_kmajor = [&](uint32_t d_tmem, uint32_t a, uint32_t b) {
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t in_chunk = (kk & 3) * 32;
          mma_ss(d_tmem, smem_desc_sw128(a + (kk >> 2) * C::CHUNK_BYTES + in_chunk, 16, 1024),
                 smem_desc_sw128(b + (kk >> 2) * C::KV_CHUNK + in_chunk, 16, 1024), IDESC_SS, kk > 0 ? 1u : 0u);
        }
      };
      bool ok = wait_bounded(smem_u32(&bars->q_full), 0, abort_flag, to, ROLE_MMA);
      ok = ok && wait_bounded(smem_u32(&bars->k_full[0]), 0, abort_flag, to, ROLE_MMA);
      if (ok) {
        tc_fence_after();
        mma_kmajor(tmem + BQ_S, sQ, sK);
        mma_commit(smem_u32(&bars->s_full));
      }
      ok = ok && wait_bounded(smem_u32(&bars->do_full), 0, abort_flag, to, ROLE_MMA);
      ok = ok && wait_bounded(smem_u32(&bars->v_full[0]), 0, abort_flag, to, ROLE_MMA);
      if (ok) {
        tc_fence_after();
        mma_kmajor(tmem + BQ_DP, sDO, sV);
        mma_commit(smem_u32(&bars->dp_full));
        mma_commit(smem_u32(&bars->v_empty[0]));
      }
      for (int j = 1; ok && j <= nkv; ++j) {
        const int i = j - 1;
        if (j < nkv) {
          const int ks = j % C::DQ_KS;
          ok = wait_bounded(smem_u32(&bars->k_full[ks]), (j / C::DQ_KS) & 1, abort_flag, to, ROLE_MMA) &&
               wait_bounded(smem_u32(&bars->s_free), i & 1, abort_flag, to, ROLE_MMA);
          if (!ok) break;
          tc_fence_after();
          mma_kmajor(tmem + BQ_S, sQ, sK + ks * C::KV_TILE);
          mma_commit(smem_u32(&bars->s_full));
        }
        ok = wait_bounded(smem_u32(&bars->ds_ready), i & 1, abort_flag, to, ROLE_MMA);
        if (!ok) break;
        tc_fence_after();
        const uint32_t kbase = sK + (i % C::DQ_KS) * C::KV_TILE;
#pragma unroll
        for (int kk = 0; kk < BNK / 16; ++kk)
          mma_ts(tmem + BQ_DQ, tmem + BQ_DP + kk * 8, smem_desc_sw128(kbase + kk * 2048, C::KV_CHUNK, 1024),
                 IDESC_DQ, (i > 0 || kk > 0) ? 1u : 0u);
        mma_commit(smem_u32(&bars->k_empty[i % C::DQ_KS]));
        if (j < nkv) {
          const int vs = j % C::DQ_VS;
          ok = wait_bounded(smem_u32(&bars->v_full[vs]), (j / C::DQ_VS) & 1, abort_flag, to, ROLE_MMA);
          if (!ok) break;
          tc_fence_after();
          mma_kmajor(tmem + BQ_DP, sDO, sV + vs * C::KV_TILE);
          mma_commit(smem_u32(&bars->dp_full));
          mma_commit(smem_u32(&bars->v_empty[vs]));
        }
      }
      mma_commit(smem_u32(&bars->mma_final));
      wait_drain(smem_u32(&bars->mma_final), 0, to);
    }
  } else {
    // ------------------------------------------------------------ elementwise warps 0..3
    const int r = threadIdx.x;
    const int row = q0 + r;
    const bool valid = row < p.N;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    // D = dO . O and -LSE*log2(e) of this row, kept in registers and written
    // to the workspace for the dK/dV kernel (padding rows: D = 0, -inf).
    // O is read row-coalesced from global memory (LPR lanes per row, 16
    // bytes each, RPI rows per load instruction, up to 16 loads of a lane in
    // flight); dO too at d = 64, and from the resident tile in shared memory
    // once its load has landed at d >= 128 (measured: the global loads win
    // at d = 64, the shared tile at d = 128).  Each row's partial dot
    // products are summed across its lanes and handed to the row's thread.
    bool ok = true;
    float dsum = 0.f;
    {
      constexpr int NV = HD / 8;              // 16-byte vectors per row
      constexpr int LPR = NV < 32 ? NV : 32;  // lanes per row
      constexpr int RPI = 32 / LPR;           // rows per load instruction
      constexpr int NI = 32 / RPI;            // load instructions per warp
      constexpr int BATCH = NI < 16 ? NI : 16;
      const int sub = lane % LPR, grp = lane / LPR;
      const uint32_t unit = static_cast<uint32_t>(sub >> 3) * C::CHUNK_BYTES;  // 64-column chunk of this lane's 16 bytes
#pragma unroll
      for (int b0 = 0; b0 < NI && ok; b0 += BATCH) {
        uint4 a[BATCH], gg[BATCH];
#pragma unroll
        for (int i = 0; i < BATCH; ++i) {
          const int rw = q0 + warp * 32 + (b0 + i) * RPI + grp;
          a[i] = gg[i] = make_uint4(0u, 0u, 0u, 0u);
          if (rw < p.N && sub * 8 < p.d) {  // columns past d (padded head dimension) are not read
            const size_t off = (static_cast<size_t>(bh) * p.N + rw) * p.d + sub * 8;
            a[i] = *reinterpret_cast<const uint4*>(p.o + off);
            if constexpr (HD == 64) gg[i] = *reinterpret_cast<const uint4*>(p.dout + off);
          }
        }
        if (HD > 64 && b0 == 0) ok = wait_warp(smem_u32(&bars->do_full), 0, abort_flag, to);
        if (!ok) break;
#pragma unroll
        for (int i = 0; i < BATCH; ++i) {
          // the tile's dO row (zero past N and past d), 128-byte swizzle
          const int rt = warp * 32 + (b0 + i) * RPI + grp;
          const uint4 g =
              (HD == 64) ? gg[i] : ld_shared_v4(sDO + unit + rt * 128 + (((sub & 7) ^ (rt & 7)) << 4));
          const uint32_t aw[4] = {a[i].x, a[i].y, a[i].z, a[i].w}, gw[4] = {g.x, g.y, g.z, g.w};
          float part = 0.f;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            part = fmaf(__uint_as_float(aw[e] << 16), __uint_as_float(gw[e] << 16), part);
            part = fmaf(__uint_as_float(aw[e] & 0xffff0000u), __uint_as_float(gw[e] & 0xffff0000u), part);
          }
#pragma unroll
          for (int m = LPR / 2; m > 0; m >>= 1) part += __shfl_xor_sync(0xffffffffu, part, m);
          const float row_sum = __shfl_sync(0xffffffffu, part, (lane % RPI) * LPR);
          if (lane / RPI == b0 + i) dsum = row_sum;
        }
      }
    }
    const float nlse2 = valid ? -p.lse[static_cast<size_t>(bh) * p.N + row] * LOG2E_F : -INFINITY;
    if (ok) {
      const size_t vrow = static_cast<size_t>(bh) * p.n_tiles * BM + q0 + r;
      p.dvec[vrow] = dsum;
      p.lse2[vrow] = nlse2;
    }

    const float c = p.scale_log2;
    for (int j = 0; ok && j < nkv; ++j) {
      ok = wait_warp(smem_u32(&bars->s_full), j & 1, abort_flag, to);
      if (!ok) break;
      tc_fence_after();
      float pr[BNK];
      {
        uint32_t s[BNK];
#pragma unroll
        for (int cc = 0; cc < BNK / 32; ++cc)
          tmem_ld32(lane_addr + BQ_S + cc * 32, *reinterpret_cast<uint32_t(*)[32]>(&s[cc * 32]));
        tmem_wait_ld();
#pragma unroll
        for (int cc = 0; cc < BNK / 32; ++cc) reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(&s[cc * 32]));
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bars->s_free));
        const int kv0 = j * BNK;
        const bool diag = CAUSAL && (kv0 + BNK - 1 > q0);  // the tile reaches past the first row
        const bool tail = !CAUSAL && (kv0 + BNK > p.N);
        const int lim = diag ? (row - kv0) : (p.N - 1 - kv0);  // last allowed key column
        bwd_probs<false, BNK, C::EMU_PAIRS>(pr, s, c, nlse2, nullptr, diag || tail, lim, false);
      }
      ok = wait_warp(smem_u32(&bars->dp_full), j & 1, abort_flag, to);
      if (!ok) break;
      tc_fence_after();
      ds_to_tmem<BNK>(lane_addr + BQ_DP, pr, nullptr, false, dsum);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars->ds_ready));
    }
    if (ok) ok = wait_warp(smem_u32(&bars->mma_final), 0, abort_flag, to);
    if (ok) {
      // Every MMA has completed, so the Q tile's buffer takes dQ (bf16, times
      // the softmax scale) for one TMA store per 64 columns; the store skips
      // rows past N and columns past d.  Only the storing thread waits
      // (bounded) for the four warps, so a warp that gave up earlier cannot
      // leave the others blocked.
      tc_fence_after();
      stage_row_bf16<HD>(sQ, lane_addr + BQ_DQ, r, p.scale);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars->epi));
      if (threadIdx.x == 0 && wait_bounded(smem_u32(&bars->epi), 0, abort_flag, to, ROLE_SOFTMAX)) {
#pragma unroll
        for (int cc = 0; cc < HD / 64; ++cc) tma_store_3d(&tm_dq, sQ + cc * C::CHUNK_BYTES, cc * 64, q0, bh);
        bulk_commit_group();
        bulk_wait_read();  // the shared-memory source must stay valid until read
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == BWD_MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

struct KvBars {
  uint64_t k_full, v_full;  // the resident K and V tiles (S^T waits for K only)
  uint64_t q_full[3], q_empty[3];
  uint64_t s_full, dp_full, p_ready, ds_ready, mma_final;
  uint64_t epi;  // the four elementwise warps staged their gradient rows in shared memory
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(KvBars) <= 256, "barrier block");

// TMEM columns of the dK/dV kernel: S^T [0,BMQ), dP^T [128,128+BMQ), and
// the accumulators from column 256: dV then dK (both gradients), or the one
// gradient of a single pass.
constexpr uint32_t BK_S = 0, BK_DP = 128, BK_DV = 256;

template <int HD, bool CAUSAL, int PASS>
__global__ void __launch_bounds__(BWD_THREADS, 1)
    fa2_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                        const __grid_constant__ CUtensorMap tm_dk, const __grid_constant__ CUtensorMap tm_dv,
                        const BwdParams p) {
  using C = BwdCfg<HD>;
  constexpr int BMQ = C::BMQ;
  constexpr bool DO_DV = PASS != BWD_KV_DK, DO_DK = PASS != BWD_KV_DV;
  static_assert(PASS == BWD_KV_BOTH ? HD <= 128 : HD == 256, "pass split only at d = 256");
  constexpr uint32_t BK_DK = (PASS == BWD_KV_BOTH) ? BK_DV + HD : BK_DV;
  int bh, kt;
  bwd_item<CAUSAL, false>(p, bh, kt);
  const int k0 = kt * BN;
  const int i_begin = CAUSAL ? k0 / BMQ : 0;  // query tiles that see this key tile
  const int nq = p.n_qtiles - i_begin;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t base = (raw_addr + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw_addr);
  KvBars* bars = reinterpret_cast<KvBars*>(smem + C::KV_OFF_BAR);
  volatile int* abort_flag = &bars->abort;
  const uint32_t sK = base + C::KV_OFF_K, sV = base + C::KV_OFF_V;
  const uint32_t sQ = base + C::KV_OFF_Q, sDO = base + C::KV_OFF_DO;
  const float* vec = reinterpret_cast<const float*>(smem + C::KV_OFF_VEC);

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bars->k_full), 1);
    mbar_init(smem_u32(&bars->v_full), 1);
    for (int s = 0; s < C::KV_QS; ++s) {
      mbar_init(smem_u32(&bars->q_full[s]), 1);
      mbar_init(smem_u32(&bars->q_empty[s]), 1);
    }
    mbar_init(smem_u32(&bars->s_full), 1);
    mbar_init(smem_u32(&bars->dp_full), 1);
    mbar_init(smem_u32(&bars->p_ready), 4);
    mbar_init(smem_u32(&bars->ds_ready), 4);
    mbar_init(smem_u32(&bars->mma_final), 1);
    mbar_init(smem_u32(&bars->epi), 4);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == BWD_MMA_WARP) {
    tmem_alloc(smem_u32(&bars->tmem_base), TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == BWD_PRODUCER_WARP && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    prefetch_tmap(&tm_do);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const unsigned long long to = p.timeout_ns;
  const size_t vec_head = static_cast<size_t>(bh) * p.n_tiles * BM;

  if (warp == BWD_PRODUCER_WARP) {
    if (lane == 0) {
      // K, then the first (Q, dO, lse2, D) stage, then V (read by dP^T
      // only; the dV pass of d = 256 does not read it).
      const uint32_t bk = smem_u32(&bars->k_full), bv = smem_u32(&bars->v_full);
      const bool load_kv = p.inject_timeout != 2;
      if (load_kv) {
        mbar_arrive_expect_tx(bk, C::TILE_BYTES);
        for (int c = 0; c < C::KCH; ++c) tma_load_3d(sK + c * C::CHUNK_BYTES, &tm_k, bk, c * 64, k0, bh);
      }
      int issued = 0;
      for (int t = 0; t < nq; ++t) {
        const int s = t % C::KV_QS;
        if (t >= C::KV_QS &&
            !wait_bounded(smem_u32(&bars->q_empty[s]), ((t / C::KV_QS) - 1) & 1, abort_flag, to, ROLE_PRODUCER))
          break;
        const int i = i_begin + t;
        const uint32_t bq = smem_u32(&bars->q_full[s]);
        mbar_arrive_expect_tx(bq, 2 * C::Q_TILE + 2 * BMQ * 4);
        for (int c = 0; c < C::KCH; ++c) {
          tma_load_3d(sQ + s * C::Q_TILE + c * C::Q_CHUNK, &tm_q, bq, c * 64, i * BMQ, bh);
          tma_load_3d(sDO + s * C::Q_TILE + c * C::Q_CHUNK, &tm_do, bq, c * 64, i * BMQ, bh);
        }
        const uint32_t sv = base + C::KV_OFF_VEC + s * 1024;
        bulk_load_1d(sv, p.lse2 + vec_head + i * BMQ, BMQ * 4, bq);
        bulk_load_1d(sv + 512, p.dvec + vec_head + i * BMQ, BMQ * 4, bq);
        if (DO_DK && t == 0 && load_kv) {
          mbar_arrive_expect_tx(bv, C::TILE_BYTES);
          for (int c = 0; c < C::KCH; ++c) tma_load_3d(sV + c * C::CHUNK_BYTES, &tm_v, bv, c * 64, k0, bh);
        }
        ++issued;
      }
      if (load_kv) {
        wait_drain(bk, 0, to);
        if (DO_DK && issued > 0) wait_drain(bv, 0, to);
      }
      for (int x = (issued > C::KV_QS ? issued - C::KV_QS : 0); x < issued; ++x)
        wait_drain(smem_u32(&bars->q_full[x % C::KV_QS]), (x / C::KV_QS) & 1, to);
    }
  } else if (warp == BWD_MMA_WARP) {
    // Both gradients: S^T(0), dP^T(0); then per query tile t: dV(t),
    // S^T(t+1), dK(t), dP^T(t+1).  dV pass: S^T(0); then dV(t), S^T(t+1).
    // dK pass: S^T(0), dP^T(0); then dK(t), S^T(t+1), dP^T(t+1).  P^T(t)
    // lives in S^T's columns and dS^T(t) in dP^T's, so each overwrite is
    // issued after the MMA that reads them (in order).
    if (lane == 0) {
      constexpr uint32_t IDESC_SS = idesc_bf16_f32(BN, BMQ, false, false);
      constexpr uint32_t IDESC_ACC = idesc_bf16_f32(BN, HD, false, true);
      // A: the 128-row K or V tile; B: a BMQ-row Q or dO tile; both K-major.
      auto mma_kmajor = [&](uint32_t d_tmem, uint32_t a, uint32_t b) {
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t in_chunk = (kk & 3) * 32;
          mma_ss(d_tmem, smem_desc_sw128(a + (kk >> 2) * C::CHUNK_BYTES + in_chunk, 16, 1024),
                 smem_desc_sw128(b + (kk >> 2) * C::Q_CHUNK + in_chunk, 16, 1024), IDESC_SS, kk > 0 ? 1u : 0u);
        }
      };
      auto mma_acc = [&](uint32_t d_tmem, uint32_t a_tmem, uint32_t b, bool acc) {
#pragma unroll
        for (int kk = 0; kk < BMQ / 16; ++kk)
          mma_ts(d_tmem, a_tmem + kk * 8, smem_desc_sw128(b + kk * 2048, C::Q_CHUNK, 1024), IDESC_ACC,
                 (acc || kk > 0) ? 1u : 0u);
      };
      bool ok = wait_bounded(smem_u32(&bars->k_full), 0, abort_flag, to, ROLE_MMA) &&
                wait_bounded(smem_u32(&bars->q_full[0]), 0, abort_flag, to, ROLE_MMA);
      if (ok) {
        tc_fence_after();
        mma_kmajor(tmem + BK_S, sK, sQ);
        mma_commit(smem_u32(&bars->s_full));
      }
      if constexpr (DO_DK) {
        ok = ok && wait_bounded(smem_u32(&bars->v_full), 0, abort_flag, to, ROLE_MMA);
        if (ok) {
          tc_fence_after();
          mma_kmajor(tmem + BK_DP, sV, sDO);
          mma_commit(smem_u32(&bars->dp_full));
        }
      }
      for (int t = 0; ok && t < nq; ++t) {
        const int s = t % C::KV_QS;
        const bool more = t + 1 < nq;
        const int s1 = (t + 1) % C::KV_QS;
        if constexpr (DO_DV) {
          ok = wait_bounded(smem_u32(&bars->p_ready), t & 1, abort_flag, to, ROLE_MMA);
          if (!ok) break;
          tc_fence_after();
          mma_acc(tmem + BK_DV, tmem + BK_S, sDO + s * C::Q_TILE, t > 0);
          // dV pass: the stage's last reader was just issued (the producer
          // may then refill it, which the next S^T waits for).
          if constexpr (PASS == BWD_KV_DV) mma_commit(smem_u32(&bars->q_empty[s]));
        } else {
          ok = wait_bounded(smem_u32(&bars->ds_ready), t & 1, abort_flag, to, ROLE_MMA);
          if (!ok) break;
          tc_fence_after();
          mma_acc(tmem + BK_DK, tmem + BK_DP, sQ + s * C::Q_TILE, t > 0);
          mma_commit(smem_u32(&bars->q_empty[s]));
        }
        if (more) {
          ok = wait_bounded(smem_u32(&bars->q_full[s1]), ((t + 1) / C::KV_QS) & 1, abort_flag, to, ROLE_MMA);
          if (!ok) break;
          tc_fence_after();
          mma_kmajor(tmem + BK_S, sK, sQ + s1 * C::Q_TILE);
          mma_commit(smem_u32(&bars->s_full));
        }
        if constexpr (PASS == BWD_KV_BOTH) {
          ok = wait_bounded(smem_u32(&bars->ds_ready), t & 1, abort_flag, to, ROLE_MMA);
          if (!ok) break;
          tc_fence_after();
          mma_acc(tmem + BK_DK, tmem + BK_DP, sQ + s * C::Q_TILE, t > 0);
          mma_commit(smem_u32(&bars->q_empty[s]));
        }
        if (DO_DK && more) {
          mma_kmajor(tmem + BK_DP, sV, sDO + s1 * C::Q_TILE);
          mma_commit(smem_u32(&bars->dp_full));
        }
      }
      mma_commit(smem_u32(&bars->mma_final));
      wait_drain(smem_u32(&bars->mma_final), 0, to);
    }
  } else {
    // ------------------------------------------------------------ elementwise warps 0..3
    const int r = threadIdx.x;
    const int key = k0 + r;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const float c = p.scale_log2;
    bool ok = true;
    for (int t = 0; t < nq; ++t) {
      const int s = t % C::KV_QS;
      const int i = i_begin + t;
      ok = wait_warp(smem_u32(&bars->s_full), t & 1, abort_flag, to) &&
           wait_warp(smem_u32(&bars->q_full[s]), (t / C::KV_QS) & 1, abort_flag, to);
      if (!ok) break;
      tc_fence_after();
      const float* l2 = vec + s * 256;  // -LSE*log2(e) of the tile's BMQ queries (-inf past N)
      const float* dd = l2 + 128;       // D of the tile's BMQ queries
      float pr[BMQ];
      {
        uint32_t sv[BMQ];
#pragma unroll
        for (int cc = 0; cc < BMQ / 32; ++cc)
          tmem_ld32(lane_addr + BK_S + cc * 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[cc * 32]));
        tmem_wait_ld();
#pragma unroll
        for (int cc = 0; cc < BMQ / 32; ++cc) reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(&sv[cc * 32]));
        // Query i*BMQ + e sees this key only if i*BMQ + e >= key.
        const int q_first = i * BMQ;
        const bool diag = CAUSAL && (q_first < k0 + BN - 1);
        bwd_probs<true, BMQ, C::EMU_PAIRS>(pr, sv, c, 0.f, l2, diag, key - q_first, true);
      }
      if constexpr (DO_DV) {
        // P^T (bf16) over the first BMQ/2 score columns, for dV += P^T dO.
#pragma unroll
        for (int h = 0; h < BMQ / 64; ++h) {
          uint32_t pk[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) pk[e] = pack_bf16x2(pr[64 * h + 2 * e], pr[64 * h + 2 * e + 1]);
          tmem_st32(lane_addr + BK_S + 32 * h, pk);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bars->p_ready));
      }
      if constexpr (DO_DK) {
        ok = wait_warp(smem_u32(&bars->dp_full), t & 1, abort_flag, to);
        if (!ok) break;
        tc_fence_after();
        ds_to_tmem<BMQ>(lane_addr + BK_DP, pr, dd, true, 0.f);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bars->ds_ready));
      }
    }
    if (ok) ok = wait_warp(smem_u32(&bars->mma_final), 0, abort_flag, to);
    if (ok) {
      // Every MMA has completed: the V tile's buffer takes dV and the K
      // tile's dK (bf16; dK times the softmax scale) for TMA stores of 64
      // columns each, which skip rows past N and columns past d.  Only the
      // storing thread waits (bounded) for the four warps.
      tc_fence_after();
      if constexpr (DO_DV) stage_row_bf16<HD>(sV, lane_addr + BK_DV, r, 1.f);
      if constexpr (DO_DK) stage_row_bf16<HD>(sK, lane_addr + BK_DK, r, p.scale);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars->epi));
      if (threadIdx.x == 0 && wait_bounded(smem_u32(&bars->epi), 0, abort_flag, to, ROLE_SOFTMAX)) {
#pragma unroll
        for (int cc = 0; cc < HD / 64; ++cc) {
          if constexpr (DO_DV) tma_store_3d(&tm_dv, sV + cc * C::CHUNK_BYTES, cc * 64, k0, bh);
          if constexpr (DO_DK) tma_store_3d(&tm_dk, sK + cc * C::CHUNK_BYTES, cc * 64, k0, bh);
        }
        bulk_commit_group();
        bulk_wait_read();  // the shared-memory sources must stay valid until read
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == BWD_MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}
