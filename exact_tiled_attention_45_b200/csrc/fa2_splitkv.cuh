// Split-K/V exact attention for few queries against many keys (decoding, or a
// prefill chunk after a cached prefix).  Included by fa2_fwd.cu inside
// namespace fa2 (one translation unit: shares the status word and helpers).
//
// The pages distinguish the initial processing of a long prompt from
// token-by-token generation, whose bottlenecks differ (iplexlaw blog
// "FlashAttention-2: making long-context attention run efficiently on GPUs",
// section "Document the implementation difference").  With few query rows the
// work is a stream over K and V (HBM-bound), and one query block per head
// leaves most SMs idle; so the keys are split into ranges processed by
// separate CTAs, each producing a partial result normalised over its own range
// with that range's logsumexp, and a second kernel merges them exactly:
//     LSE = ln sum_s exp(LSE_s),   O = sum_s exp(LSE_s - LSE) O_s.
// Query row i sits at sequence position Nk - Nq + i (the last Nq positions);
// causal masking excludes keys after that position.
//
// With a single range the partial kernel writes the final bf16 O and LSE
// itself and no merge runs.
//
// Partial kernel: one CTA per (128-row query tile, batch*head, key range);
// 192 threads: warps 0-3 softmax (thread r <-> row r <-> TMEM lane r), warp 4
// TMA producer, warp 5 MMA issuer.  TMEM: two score buffers (the next S is
// computed while the softmax works on the current one), two P buffers (the
// softmax writes P(j+1) while P V(j) still reads P(j); it waits for P V(j)
// only to rescale O), and O.  Rows past Nq are computed on zero queries and
// never stored.
//
// Quarter mode (QUAD, at most 32 query rows, d <= 128): the query rows are
// loaded four times, into TMEM lane quadrants 0, 32, 64 and 96, so every
// softmax warp holds all of them, and warp w takes key columns 32w..32w+31 of
// each tile: a quarter of the exponentials per warp instead of all 128
// columns on the one warp whose lanes hold the rows.  Each warp keeps its own
// running max and sum; its P row is zero outside its key columns, so PV
// accumulates in quadrant w exactly the partial output of those keys.  At the
// end the four partials merge exactly (the same formula as the ranges) through
// shared memory.
//
// Head dimension 256 (also served to the square entry point as one range with
// Nq = Nk): 64-key tiles, so that a 256-column O accumulator, two score
// buffers and P fit the 512 TMEM columns and two stages of K and V fit shared
// memory next to the 64 KB query tile.

constexpr int SKV_THREADS = 192;
constexpr int SKV_PRODUCER_WARP = 4;
constexpr int SKV_MMA_WARP = 5;

// Slim configuration (d = 64, quarter mode): 2-stage K and V rings (80 KB
// of shared memory with the query tile), one score and one P buffer (256
// TMEM columns), so that two CTAs share an SM and one's set-up, hand-offs
// and tail overlap the other's stream of keys.
#ifndef FA2_SKV_SLIM_D64
#define FA2_SKV_SLIM_D64 1
#endif
template <int HD, bool QUAD>
__host__ __device__ constexpr bool skv_slim() {
  return FA2_SKV_SLIM_D64 && HD == 64 && QUAD;
}

template <int HD, bool SLIM = false>
struct SkvCfg {
  static constexpr int SBN = (HD == 256) ? 64 : 128;  // keys per tile
  static constexpr int KCH = HD / 64;                 // 64-column (128-byte) chunks
  static constexpr int Q_CHUNK = 128 * 128;           // 128 query rows x 128 bytes
  static constexpr int KV_CHUNK = SBN * 128;          // SBN key rows x 128 bytes
  static constexpr int Q_BYTES = KCH * Q_CHUNK;
  static constexpr int KV_BYTES = KCH * KV_CHUNK;
  // Deep K/V rings: the stream over keys is the bound for few queries, so
  // keep many tiles in flight (224 KB of rings for d = 128, 128 KB for d = 64,
  // 128 KB for d = 256).
  static constexpr int KS = SLIM ? 2 : (HD == 64) ? 4 : (HD == 128 ? 3 : 2);
  static constexpr int VS = KS;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + KS * KV_BYTES;
  static constexpr int OFF_BAR = OFF_V + VS * KV_BYTES;
  static constexpr int SMEM_BYTES = OFF_BAR + 256 + 1024;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(!SLIM || 2 * (SMEM_BYTES + 1024) <= 233472, "two slim CTAs per SM");
  static constexpr int MIN_BLOCKS = SLIM ? 2 : 1;  // CTAs per SM
  static constexpr int NSB = SLIM ? 1 : 2;          // score buffers
  static constexpr int NPB = SLIM ? 1 : 2;          // P buffers
  // TMEM columns: S0, S1 (SBN each), P0, P1 (SBN/2 packed bf16 pairs each), O (HD);
  // slim: S, P, O in 256 columns.
  static constexpr uint32_t TMEM_ALLOC = SLIM ? 256 : 512;
  static constexpr uint32_t TM_S0 = 0, TM_S1 = SLIM ? 0 : SBN, TM_P = NSB * SBN;
  static constexpr uint32_t TM_O = SLIM ? TM_P + SBN / 2 : (HD == 256) ? 256 : 384;
  __host__ __device__ static constexpr uint32_t tm_p(int b) { return TM_P + static_cast<uint32_t>(b) * (SBN / 2); }
  static_assert(TM_P + NPB * SBN / 2 <= TM_O && TM_O + HD <= TMEM_ALLOC, "TMEM budget");
};

struct SkvParams {
  float* o_part;    // [n_splits, B*H, Nq, d] fp32, normalised within the range
  float* lse_part;  // [n_splits, B*H, Nq] fp32 natural-log logsumexp of the range
  __nv_bfloat16* o; // final outputs, written directly when there is one range
  float* lse;
  int direct;       // 1: one range, no merge step
  int Nq;
  int Nk;
  int d;  // head dimension of q, k, v, o (<= HD; tiles are zero-padded to HD)
  int BH;
  int n_kv_tiles;       // ceil(Nk / SBN)
  int tiles_per_split;  // key tiles per range
  float scale_log2;
  unsigned long long timeout_ns;
  int inject_timeout;  // test hook: withhold the query load so the waits on it run out
};

struct SkvBarriers {
  uint64_t q_full;
  uint64_t k_full[4], k_empty[4];
  uint64_t v_full[4], v_empty[4];
  uint64_t s_full[2], s_free[2];
  uint64_t p_full[2];   // P buffer b written (by all four softmax warps)
  uint64_t pv_done[2];  // the P V MMA reading P buffer b complete
  uint64_t mma_final;
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(SkvBarriers) <= 256, "barrier block");

template <int HD, bool CAUSAL, bool QUAD>
__global__ void __launch_bounds__(SKV_THREADS, (SkvCfg<HD, skv_slim<HD, QUAD>()>::MIN_BLOCKS))
    fa2_splitkv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const SkvParams p) {
  using C = SkvCfg<HD, skv_slim<HD, QUAD>()>;
  static_assert(!QUAD || C::SBN == 128, "quarter mode needs 128-key tiles");
  const int q_first = static_cast<int>(blockIdx.x) * BM;
  const int bh = static_cast<int>(blockIdx.y);
  const int split = static_cast<int>(blockIdx.z);
  const int offset = p.Nk - p.Nq;  // sequence position of query row 0
  // Key tiles this query tile needs: all of them, or (causal) up to the
  // position of its last row.
  int n_need = p.n_kv_tiles;
  if (CAUSAL) n_need = min(n_need, (offset + min(q_first + BM, p.Nq) - 1) / C::SBN + 1);
  const int kt_begin = split * p.tiles_per_split;
  const int kt_end = min(kt_begin + p.tiles_per_split, n_need);
  const int nkv = kt_end - kt_begin;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (nkv <= 0) {
    // Nothing of this range is visible to this tile: an empty partial.
    if (warp < 4) {
      const int row = q_first + warp * 32 + lane;
      if (row < p.Nq) {
        const size_t prow = (static_cast<size_t>(split) * p.BH + bh) * p.Nq + row;
        p.lse_part[prow] = -INFINITY;
        float4* dst = reinterpret_cast<float4*>(p.o_part + prow * HD);
#pragma unroll
        for (int c = 0; c < HD / 4; ++c) dst[c] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    return;
  }

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t base = (raw_addr + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw_addr);
  SkvBarriers* bars = reinterpret_cast<SkvBarriers*>(smem + C::OFF_BAR);
  volatile int* abort_flag = &bars->abort;
  const uint32_t sQ = base + C::OFF_Q;
  const uint32_t sK = base + C::OFF_K;
  const uint32_t sV = base + C::OFF_V;
  const uint32_t b_q = smem_u32(&bars->q_full);
  const uint32_t b_final = smem_u32(&bars->mma_final);

  if (threadIdx.x == 0) {
    mbar_init(b_q, 1);
    for (int s = 0; s < C::KS; ++s) {
      mbar_init(smem_u32(&bars->k_full[s]), 1);
      mbar_init(smem_u32(&bars->k_empty[s]), 1);
    }
    for (int s = 0; s < C::VS; ++s) {
      mbar_init(smem_u32(&bars->v_full[s]), 1);
      mbar_init(smem_u32(&bars->v_empty[s]), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(smem_u32(&bars->s_full[s]), 1);
      mbar_init(smem_u32(&bars->s_free[s]), 4);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&bars->p_full[b]), 4);
      mbar_init(smem_u32(&bars->pv_done[b]), 1);
    }
    mbar_init(b_final, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == SKV_MMA_WARP) {
    tmem_alloc(smem_u32(&bars->tmem_base), C::TMEM_ALLOC);
    tmem_relinquish();
  }
  if (warp == SKV_PRODUCER_WARP && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const unsigned long long to = p.timeout_ns;

  if (warp == SKV_PRODUCER_WARP) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const bool load_q = !p.inject_timeout;
      if (load_q) {
        mbar_arrive_expect_tx(b_q, C::Q_BYTES);
        if constexpr (QUAD) {
          // Four copies of the (at most 32) query rows, 32-row boxes, at rows
          // 0, 32, 64, 96 of the tile; rows past Nq are zero-filled.
          for (int w = 0; w < 4; ++w)
            for (int c = 0; c < C::KCH; ++c)
              tma_load_3d(sQ + c * C::Q_CHUNK + w * 32 * 128, &tm_q, b_q, c * 64, 0, bh);
        } else {
          for (int c = 0; c < C::KCH; ++c) tma_load_3d(sQ + c * C::Q_CHUNK, &tm_q, b_q, c * 64, q_first, bh);
        }
      }
      int k_issued = 0, v_issued = 0;
      for (int j = 0; j < nkv; ++j) {
        const int kv0 = (kt_begin + j) * C::SBN;
        const int ks = j % C::KS;
        if (j >= C::KS &&
            !wait_bounded(smem_u32(&bars->k_empty[ks]), ((j / C::KS) - 1) & 1, abort_flag, to, ROLE_PRODUCER))
          break;
        const uint32_t kb = smem_u32(&bars->k_full[ks]);
        mbar_arrive_expect_tx(kb, C::KV_BYTES);
        for (int c = 0; c < C::KCH; ++c)
          tma_load_3d(sK + ks * C::KV_BYTES + c * C::KV_CHUNK, &tm_k, kb, c * 64, kv0, bh);
        ++k_issued;
        const int vs = j % C::VS;
        if (j >= C::VS &&
            !wait_bounded(smem_u32(&bars->v_empty[vs]), ((j / C::VS) - 1) & 1, abort_flag, to, ROLE_PRODUCER))
          break;
        const uint32_t vb = smem_u32(&bars->v_full[vs]);
        mbar_arrive_expect_tx(vb, C::KV_BYTES);
        for (int c = 0; c < C::KCH; ++c)
          tma_load_3d(sV + vs * C::KV_BYTES + c * C::KV_CHUNK, &tm_v, vb, c * 64, kv0, bh);
        ++v_issued;
      }
      if (load_q) wait_drain(b_q, 0, to);
      for (int x = (k_issued > C::KS ? k_issued - C::KS : 0); x < k_issued; ++x)
        wait_drain(smem_u32(&bars->k_full[x % C::KS]), (x / C::KS) & 1, to);
      for (int x = (v_issued > C::VS ? v_issued - C::VS : 0); x < v_issued; ++x)
        wait_drain(smem_u32(&bars->v_full[x % C::VS]), (x / C::VS) & 1, to);
    }
  } else if (warp == SKV_MMA_WARP) {
    // ------------------------------------------------------------ MMA issuer
    // Order S(0), S(1), PV(0), S(2), PV(1), ...: the next scores are computed
    // while the softmax works on the current ones.
    if (lane == 0) {
      constexpr uint32_t IDESC_S = idesc_bf16_f32(BM, C::SBN, false, false);
      constexpr uint32_t IDESC_PV = idesc_bf16_f32(BM, HD, false, true);
      bool ok = wait_bounded(b_q, 0, abort_flag, to, ROLE_MMA);
      for (int j = 0; ok && j <= nkv; ++j) {
        if (j < nkv) {
          const int ks = j % C::KS;
          const int sb = j % C::NSB;
          if (!wait_bounded(smem_u32(&bars->k_full[ks]), (j / C::KS) & 1, abort_flag, to, ROLE_MMA)) break;
          if (j >= C::NSB &&
              !wait_bounded(smem_u32(&bars->s_free[sb]), ((j - C::NSB) / C::NSB) & 1, abort_flag, to, ROLE_MMA))
            break;
          tc_fence_after();
          const uint32_t d_s = tmem + (sb ? C::TM_S1 : C::TM_S0);
          const uint32_t kbase = sK + ks * C::KV_BYTES;
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk) {
            const uint32_t in_chunk = (kk & 3) * 32;
            mma_ss(d_s, smem_desc_sw128(sQ + (kk >> 2) * C::Q_CHUNK + in_chunk, 16, 1024),
                   smem_desc_sw128(kbase + (kk >> 2) * C::KV_CHUNK + in_chunk, 16, 1024), IDESC_S, kk > 0 ? 1u : 0u);
          }
          mma_commit(smem_u32(&bars->s_full[sb]));
          mma_commit(smem_u32(&bars->k_empty[ks]));
        }
        if (j >= 1) {
          const int i = j - 1;
          const int vs = i % C::VS;
          const int pb = i % C::NPB;
          if (!wait_bounded(smem_u32(&bars->p_full[pb]), (i / C::NPB) & 1, abort_flag, to, ROLE_MMA)) break;
          if (!wait_bounded(smem_u32(&bars->v_full[vs]), (i / C::VS) & 1, abort_flag, to, ROLE_MMA)) break;
          tc_fence_after();
          const uint32_t vbase = sV + vs * C::KV_BYTES;
#pragma unroll
          for (int kk = 0; kk < C::SBN / 16; ++kk)
            mma_ts(tmem + C::TM_O, tmem + C::tm_p(pb) + kk * 8,
                   smem_desc_sw128(vbase + kk * 2048, C::KV_CHUNK, 1024), IDESC_PV, (i > 0 || kk > 0) ? 1u : 0u);
          mma_commit(smem_u32(&bars->v_empty[vs]));
          mma_commit(smem_u32(&bars->pv_done[pb]));
        }
      }
      mma_commit(b_final);
      wait_drain(b_final, 0, to);
    }
  } else if constexpr (QUAD) {
    // ------------------------------------------------------------ softmax warps 0..3, quarter mode
    const int qrow = lane;  // query row of this thread (each warp holds a copy)
    const int pos = offset + qrow;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const int col0 = warp * 32;  // this warp's key columns of every tile
    const float c_log2 = p.scale_log2;
    const uint64_t cc = f2_pack(c_log2, c_log2);
    {
      // P of the other warps' keys stays zero in this warp's lanes.
      uint32_t z[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) z[e] = 0u;
      tmem_st32(lane_addr + C::tm_p(0), z);
      tmem_st32(lane_addr + C::tm_p(0) + 32, z);
      if constexpr (C::NPB == 2) {
        tmem_st32(lane_addr + C::tm_p(1), z);
        tmem_st32(lane_addr + C::tm_p(1) + 32, z);
      }
      tmem_wait_st();
    }
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int i = 0; i < nkv; ++i) {
      const int sb = i % C::NSB;
      ok = wait_warp(smem_u32(&bars->s_full[sb]), (i / C::NSB) & 1, abort_flag, to);
      if (!ok) break;
      tc_fence_after();
      const int kv0 = (kt_begin + i) * C::SBN + col0;
      uint32_t s[32];
      tmem_ld32(lane_addr + (sb ? C::TM_S1 : C::TM_S0) + col0, s);
      tmem_wait_ld();
      reg_fence32(s);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars->s_free[sb]));
      const int lim = CAUSAL ? min(pos, p.Nk - 1) - kv0 : p.Nk - 1 - kv0;
      if (lim < 31) {
#pragma unroll
        for (int e = 0; e < 32; ++e)
          if (e > lim) s[e] = __float_as_uint(-INFINITY);
      }
      float mx4[4];
#pragma unroll
      for (int a = 0; a < 4; ++a) mx4[a] = __uint_as_float(s[a]);
#pragma unroll
      for (int e = 4; e + 8 <= 32; e += 8)  // columns 4 .. 27
#pragma unroll
        for (int a = 0; a < 4; ++a) mx4[a] = fmax3(mx4[a], __uint_as_float(s[e + a]), __uint_as_float(s[e + 4 + a]));
#pragma unroll
      for (int a = 0; a < 4; ++a) mx4[a] = fmaxf(mx4[a], __uint_as_float(s[28 + a]));  // the last 4
      const float mx = fmaxf(fmax3(mx4[0], mx4[1], mx4[2]), mx4[3]);
      const float m_cand = mx * c_log2;
      float m_new = m;
      if (m_cand > m + RESCALE_THRESHOLD) m_new = m_cand;
      const bool rescale = (i > 0) && (m_new != m);
      const float alpha = rescale ? ex2(m - m_new) : 1.f;
      const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
      const uint64_t mm = f2_pack(-m_use, -m_use);
      uint64_t acc[4] = {0, 0, 0, 0};
      uint32_t pk[16];
#pragma unroll
      for (int e = 0; e < 32; e += 2) {
        const uint64_t x = f2_fma(f2_pack(__uint_as_float(s[e]), __uint_as_float(s[e + 1])), cc, mm);
        float x0, x1;
        f2_unpack(x, x0, x1);
        const float p0 = ex2(x0), p1 = ex2(x1);
        acc[(e >> 1) & 3] = f2_add(acc[(e >> 1) & 3], f2_pack(p0, p1));
        pk[e >> 1] = pack_bf16x2(p0, p1);
      }
      float r0, r1, r2, r3;
      f2_unpack(f2_add(acc[0], acc[1]), r0, r1);
      f2_unpack(f2_add(acc[2], acc[3]), r2, r3);
      const float rowsum = (r0 + r1) + (r2 + r3);
      const int pb = i % C::NPB;
      // P buffer pb was last read by PV(i - NPB); O is accumulated by
      // PV(i-1), which must be complete only when O is rescaled here (with one
      // P buffer the first wait already covers it).
      if (i >= C::NPB) {
        ok = wait_warp(smem_u32(&bars->pv_done[pb]), ((i - C::NPB) / C::NPB) & 1, abort_flag, to);
        if (!ok) break;
        tc_fence_after();
      }
      if (i > 0 && __any_sync(0xffffffffu, rescale)) {
        if constexpr (C::NPB == 2) {
          ok = wait_warp(smem_u32(&bars->pv_done[pb ^ 1]), ((i - 1) >> 1) & 1, abort_flag, to);
          if (!ok) break;
          tc_fence_after();
        }
        {
          const uint64_t aa = f2_pack(alpha, alpha);
#pragma unroll
          for (int c = 0; c < HD / 32; ++c) {
            uint32_t o[32];
            tmem_ld32(lane_addr + C::TM_O + c * 32, o);
            tmem_wait_ld();
            reg_fence32(o);
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              float a0, a1;
              f2_unpack(f2_mul(f2_pack(__uint_as_float(o[e]), __uint_as_float(o[e + 1])), aa), a0, a1);
              o[e] = __float_as_uint(a0);
              o[e + 1] = __float_as_uint(a1);
            }
            tmem_st32(lane_addr + C::TM_O + c * 32, o);
          }
        }
      }
      tmem_st16(lane_addr + C::tm_p(pb) + 16 * warp, pk);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars->p_full[pb]));
      l = l * alpha + rowsum;
      m = m_new;
    }
    if (ok) ok = wait_warp(smem_u32(&bars->pv_done[(nkv - 1) % C::NPB]), ((nkv - 1) / C::NPB) & 1, abort_flag, to);
    // Merge of the four quarters.  Every softmax warp reaches both named
    // barriers whatever happened above (after a time-out the values are
    // unspecified, as documented, but no warp is left waiting).  The K and V
    // rings are idle here: their last readers, the final S and P V MMAs,
    // completed before the final pv_done.
    constexpr int OST = HD + 4;  // padded row stride (floats) of the exchange buffer
    constexpr int XO_BYTES = 4 * 32 * OST * 4;
    float* xo = reinterpret_cast<float*>(smem + C::OFF_K);             // [4 warps][32 rows][OST]
    float* xm = reinterpret_cast<float*>(smem + C::OFF_K + XO_BYTES);  // [4][32] running max (log2)
    float* xl = xm + 128;                                              // [4][32] running sum
    static_assert(C::OFF_K + XO_BYTES + 2 * 128 * 4 <= C::OFF_BAR, "exchange buffer");
    xm[warp * 32 + lane] = m;
    xl[warp * 32 + lane] = l;
    named_barrier(1, 128);
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) M = fmaxf(M, xm[w * 32 + lane]);
    float L = 0.f, wt_self = 0.f;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const float mw = xm[w * 32 + lane];
      const float wt = (mw == -INFINITY) ? 0.f : ex2(mw - M);
      L += wt * xl[w * 32 + lane];
      if (w == warp) wt_self = wt;
    }
    const float f_self = (L > 0.f) ? wt_self / L : 0.f;
    tc_fence_after();
#pragma unroll
    for (int c = 0; c < HD / 32; ++c) {
      uint32_t o[32];
      tmem_ld32(lane_addr + C::TM_O + c * 32, o);
      tmem_wait_ld();
      reg_fence32(o);
      float4* dst = reinterpret_cast<float4*>(xo + (warp * 32 + lane) * OST + c * 32);
#pragma unroll
      for (int e = 0; e < 32; e += 4)
        dst[e / 4] = make_float4(__uint_as_float(o[e]) * f_self, __uint_as_float(o[e + 1]) * f_self,
                                 __uint_as_float(o[e + 2]) * f_self, __uint_as_float(o[e + 3]) * f_self);
    }
    named_barrier(1, 128);
    if (ok && qrow < p.Nq) {
      // Warp w sums columns [w*HD/4, (w+1)*HD/4) of this thread's row.
      constexpr int CW = HD / 4;
      const int cb = warp * CW;
      const size_t prow = (static_cast<size_t>(split) * p.BH + bh) * p.Nq + qrow;
#pragma unroll
      for (int c = 0; c < CW; c += 8) {
        float v8[8];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            const float4 b = *reinterpret_cast<const float4*>(xo + (w * 32 + qrow) * OST + cb + c + 4 * h);
            a.x += b.x;
            a.y += b.y;
            a.z += b.z;
            a.w += b.w;
          }
          v8[4 * h] = a.x;
          v8[4 * h + 1] = a.y;
          v8[4 * h + 2] = a.z;
          v8[4 * h + 3] = a.w;
        }
        if (p.direct) {
          if (cb + c < p.d)
            *reinterpret_cast<uint4*>(p.o + prow * p.d + cb + c) =
                make_uint4(pack_bf16x2(v8[0], v8[1]), pack_bf16x2(v8[2], v8[3]), pack_bf16x2(v8[4], v8[5]),
                           pack_bf16x2(v8[6], v8[7]));
        } else {
          float4* dst = reinterpret_cast<float4*>(p.o_part + prow * HD + cb + c);
          dst[0] = make_float4(v8[0], v8[1], v8[2], v8[3]);
          dst[1] = make_float4(v8[4], v8[5], v8[6], v8[7]);
        }
      }
      if (warp == 0) {
        const float lse_row = (L > 0.f) ? (M + log2f(L)) * 0.69314718055994531f : -INFINITY;
        if (p.direct)
          p.lse[prow] = lse_row;
        else
          p.lse_part[prow] = lse_row;
      }
    }
  } else {
    // ------------------------------------------------------------ softmax warps 0..3
    const int r = threadIdx.x;
    const int row = q_first + r;
    const int pos = offset + row;  // sequence position of this query row
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const float c_log2 = p.scale_log2;
    const uint64_t cc = f2_pack(c_log2, c_log2);
    // A warp whose 32 rows are all past Nq has nothing to store: it only
    // keeps the hand-offs going.
    const bool live = q_first + warp * 32 < p.Nq;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int i = 0; i < nkv; ++i) {
      const int sb = i % C::NSB;
      ok = wait_warp(smem_u32(&bars->s_full[sb]), (i / C::NSB) & 1, abort_flag, to);
      if (!ok) break;
      tc_fence_after();
      constexpr int SBN = C::SBN;
      const int kv0 = (kt_begin + i) * SBN;
      uint32_t pk[SBN / 64][32];
      float alpha = 1.f, rowsum = 0.f, m_new = m;
      bool rescale = false;
      if (live) {
        uint32_t s[SBN];
        const uint32_t s_addr = lane_addr + (sb ? C::TM_S1 : C::TM_S0);
#pragma unroll
        for (int c = 0; c < SBN / 32; ++c)
          tmem_ld32(s_addr + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&s[c * 32]));
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < SBN / 32; ++c) reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(&s[c * 32]));
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bars->s_free[sb]));
        // Mask: keys past the row's position (causal) or past Nk.
        const int lim = CAUSAL ? min(pos, p.Nk - 1) - kv0 : p.Nk - 1 - kv0;
        if (lim < SBN - 1) {
#pragma unroll
          for (int e = 0; e < SBN; ++e)
            if (e > lim) s[e] = __float_as_uint(-INFINITY);
        }
        float mx8[8];
#pragma unroll
        for (int a = 0; a < 8; ++a) mx8[a] = __uint_as_float(s[a]);
#pragma unroll
        for (int e = 8; e + 16 <= SBN; e += 16)  // columns 8 .. SBN-9
#pragma unroll
          for (int a = 0; a < 8; ++a)
            mx8[a] = fmax3(mx8[a], __uint_as_float(s[e + a]), __uint_as_float(s[e + 8 + a]));
#pragma unroll
        for (int a = 0; a < 8; ++a) mx8[a] = fmaxf(mx8[a], __uint_as_float(s[SBN - 8 + a]));  // the last 8
        const float mx = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]));
        const float m_cand = mx * c_log2;
        if (m_cand > m + RESCALE_THRESHOLD) m_new = m_cand;
        rescale = (i > 0) && (m_new != m);
        alpha = rescale ? ex2(m - m_new) : 1.f;
        const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
        const uint64_t mm = f2_pack(-m_use, -m_use);
        uint64_t acc[4] = {0, 0, 0, 0};
#pragma unroll
        for (int c = 0; c < SBN / 32; ++c) {
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const uint64_t x =
                f2_fma(f2_pack(__uint_as_float(s[c * 32 + e]), __uint_as_float(s[c * 32 + e + 1])), cc, mm);
            float x0, x1;
            f2_unpack(x, x0, x1);
            const float p0 = ex2(x0), p1 = ex2(x1);
            acc[(e >> 1) & 3] = f2_add(acc[(e >> 1) & 3], f2_pack(p0, p1));
            pk[c >> 1][(c & 1) * 16 + (e >> 1)] = pack_bf16x2(p0, p1);
          }
        }
        float r0, r1, r2, r3;
        f2_unpack(f2_add(acc[0], acc[1]), r0, r1);
        f2_unpack(f2_add(acc[2], acc[3]), r2, r3);
        rowsum = (r0 + r1) + (r2 + r3);
      } else {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bars->s_free[sb]));
      }
      const int pb = i % C::NPB;
      // P buffer pb was last read by PV(i - NPB); O is accumulated by
      // PV(i-1), which must be complete only when O is rescaled here (with one
      // P buffer the first wait already covers it).
      if (i >= C::NPB) {
        ok = wait_warp(smem_u32(&bars->pv_done[pb]), ((i - C::NPB) / C::NPB) & 1, abort_flag, to);
        if (!ok) break;
        tc_fence_after();
      }
      if (i > 0 && live && __any_sync(0xffffffffu, rescale)) {
        if constexpr (C::NPB == 2) {
          ok = wait_warp(smem_u32(&bars->pv_done[pb ^ 1]), ((i - 1) >> 1) & 1, abort_flag, to);
          if (!ok) break;
          tc_fence_after();
        }
        {
          const uint64_t aa = f2_pack(alpha, alpha);
#pragma unroll
          for (int c = 0; c < HD / 32; ++c) {
            uint32_t o[32];
            tmem_ld32(lane_addr + C::TM_O + c * 32, o);
            tmem_wait_ld();
            reg_fence32(o);
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              float a0, a1;
              f2_unpack(f2_mul(f2_pack(__uint_as_float(o[e]), __uint_as_float(o[e + 1])), aa), a0, a1);
              o[e] = __float_as_uint(a0);
              o[e + 1] = __float_as_uint(a1);
            }
            tmem_st32(lane_addr + C::TM_O + c * 32, o);
          }
        }
      }
      if (live) {
#pragma unroll
        for (int h = 0; h < SBN / 64; ++h) tmem_st32(lane_addr + C::tm_p(pb) + 32 * h, pk[h]);
        tmem_wait_st();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars->p_full[pb]));
      l = l * alpha + rowsum;
      m = m_new;
    }
    if (ok) ok = wait_warp(smem_u32(&bars->pv_done[(nkv - 1) % C::NPB]), ((nkv - 1) / C::NPB) & 1, abort_flag, to);
    if (ok && live) {
      tc_fence_after();
      const bool store = row < p.Nq;
      const size_t prow = (static_cast<size_t>(split) * p.BH + bh) * p.Nq + row;
      const float inv_l = (l > 0.f) ? 1.f / l : 0.f;
      // 32 columns at a time (a 256-column O does not fit in registers).
#pragma unroll
      for (int c = 0; c < HD / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(lane_addr + C::TM_O + c * 32, o);
        tmem_wait_ld();
        reg_fence32(o);
        if (!store) continue;
        if (p.direct) {
          // One range: this is the final result (prow = bh * Nq + row).
          if (c * 32 < p.d) {
            uint4* dst = reinterpret_cast<uint4*>(p.o + prow * p.d + c * 32);
#pragma unroll
            for (int e = 0; e < 32; e += 8)
              dst[e / 8] = make_uint4(pack_bf16x2(__uint_as_float(o[e]) * inv_l, __uint_as_float(o[e + 1]) * inv_l),
                                      pack_bf16x2(__uint_as_float(o[e + 2]) * inv_l, __uint_as_float(o[e + 3]) * inv_l),
                                      pack_bf16x2(__uint_as_float(o[e + 4]) * inv_l, __uint_as_float(o[e + 5]) * inv_l),
                                      pack_bf16x2(__uint_as_float(o[e + 6]) * inv_l, __uint_as_float(o[e + 7]) * inv_l));
          }
        } else {
          float4* dst = reinterpret_cast<float4*>(p.o_part + prow * HD + c * 32);
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            dst[e / 4] = make_float4(__uint_as_float(o[e]) * inv_l, __uint_as_float(o[e + 1]) * inv_l,
                                     __uint_as_float(o[e + 2]) * inv_l, __uint_as_float(o[e + 3]) * inv_l);
        }
      }
      if (store) {
        const float lse_row = (l > 0.f) ? (m + log2f(l)) * 0.69314718055994531f : -INFINITY;
        if (p.direct)
          p.lse[prow] = lse_row;
        else
          p.lse_part[prow] = lse_row;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == SKV_MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_ALLOC);
  }
}

// Merge of the partial results: one warp per query row; lane l holds
// columns [l*HD/32, (l+1)*HD/32).
template <int HD>
__global__ void __launch_bounds__(128) fa2_splitkv_combine_kernel(const float* __restrict__ o_part,
                                                                  const float* __restrict__ lse_part,
                                                                  __nv_bfloat16* __restrict__ o, float* __restrict__ lse,
                                                                  int rows, int n_splits, int d) {
  const int row = static_cast<int>(blockIdx.x) * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  constexpr int PER = HD / 32;  // 8 (d = 256), 4 (d = 128) or 2 (d = 64) columns per lane
  float mx = -INFINITY;
  for (int s = 0; s < n_splits; ++s) mx = fmaxf(mx, lse_part[static_cast<size_t>(s) * rows + row]);
  float acc[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) acc[e] = 0.f;
  float wsum = 0.f;
  if (mx != -INFINITY) {
    for (int s = 0; s < n_splits; ++s) {
      const float ls = lse_part[static_cast<size_t>(s) * rows + row];
      if (ls == -INFINITY) continue;  // a range with no visible key
      const float w = __expf(ls - mx);
      wsum += w;
      const float* src = o_part + (static_cast<size_t>(s) * rows + row) * HD + lane * PER;
      if constexpr (PER >= 4) {
#pragma unroll
        for (int q4 = 0; q4 < PER / 4; ++q4) {
          const float4 x = *reinterpret_cast<const float4*>(src + 4 * q4);
          acc[4 * q4] += w * x.x;
          acc[4 * q4 + 1] += w * x.y;
          acc[4 * q4 + 2] += w * x.z;
          acc[4 * q4 + 3] += w * x.w;
        }
      } else {
        const float2 x = *reinterpret_cast<const float2*>(src);
        acc[0] += w * x.x;
        acc[1] += w * x.y;
      }
    }
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  __nv_bfloat16* dst = o + static_cast<size_t>(row) * d + lane * PER;
  if (lane * PER >= d) {
    // columns of the zero padding up to HD: nothing to store
  } else if constexpr (PER == 8) {
    *reinterpret_cast<uint4*>(dst) = make_uint4(pack_bf16x2(acc[0] * inv, acc[1] * inv), pack_bf16x2(acc[2] * inv, acc[3] * inv),
                                                pack_bf16x2(acc[4] * inv, acc[5] * inv), pack_bf16x2(acc[6] * inv, acc[7] * inv));
  } else if constexpr (PER == 4) {
    *reinterpret_cast<uint2*>(dst) = make_uint2(pack_bf16x2(acc[0] * inv, acc[1] * inv),
                                                pack_bf16x2(acc[2] * inv, acc[3] * inv));
  } else {
    *reinterpret_cast<uint32_t*>(dst) = pack_bf16x2(acc[0] * inv, acc[1] * inv);
  }
  if (lane == 0) lse[row] = (wsum > 0.f) ? mx + logf(wsum) : -INFINITY;
}
