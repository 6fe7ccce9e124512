// Backward pass of exact attention on sm_100a: dQ, dK, dV from Q, K, V, dO,
// the forward's LSE and D_i = rowsum(dO_i * O_i).
//
// The pages name the backward only by its method: tiling and recomputation,
// the attention matrix is rebuilt from Q, K and the stored softmax statistics
// instead of being kept (Flash Attention | Hermes Skill, "Quick start";
// FlashAttention-3 runs FP16/BF16 forward and backward, same pages, "Workflow
// 3: H100 FP8 optimization (FlashAttention-3)").  With S = scale Q K^T and
// P = exp(S - LSE) recomputed per (query block, key block):
//     dV = P^T dO,  dP = dO V^T,  dS = P * (dP - D),  dQ = scale dS K,
//     dK = scale dS^T Q,   D_i = sum_d dO_id O_id = sum_j P_ij dP_ij.
//
// Two kernels after a prologue that forms D_i.  The dK/dV kernel runs one
// CTA per (batch, head, 128-key block): K_j and V_j stay in shared memory and
// dK_j, dV_j accumulate in tensor memory over the query blocks that see the
// keys.  The dQ kernel runs one CTA per (batch, head, 128-query block): Q_i
// and dO_i stay in shared memory and dQ_i accumulates in tensor memory over
// the key blocks the queries see.  Each recomputes S, P, dP and dS for its
// blocks; computing dQ on its own costs three more products per block pair
// than adding dQ partials from the dK/dV kernel into a shared buffer, and
// measured on B200 it is far cheaper: those partials, 64 KB per 128x128
// block pair, were bounded by the L2's reduction throughput.
//
// dK/dV kernel: scores are computed transposed (keys on the TMEM lanes).
// P^T, written back into tensor memory over S^T by the gradient warps (after
// each has read its whole half row of S^T), is the A operand of
// dV += P^T dO; dS^T goes to shared memory in the 128-byte-swizzled layout,
// read K-major as the A operand of dK += dS^T Q.  Tensor memory: S^T [0,128)
// with P^T (16-bit) over [64,128), dP^T [128,256), dV [256,256+D),
// dK [256+D,256+2D).
//
// dQ kernel: queries on the lanes, like the forward: S [0,128), dP [128,256),
// dS (16-bit) written over S's upper half [64,128) as the A operand of
// dQ += dS K, dQ [256,256+D).
#pragma once

namespace fa {

struct BwdParams {
  void* dk;                 // [B, N_k, H, D], 16-bit like the inputs
  void* dv;                 // [B, N_k, H, D]
  void* dq;                 // [B, N_q, H, D]
  const float* lse;         // [B, H, N_q] natural log (forward output)
  const float* delta;       // [B, H, N_q] rowsum(dO * O)
  int B, Nq, Nk, H;
  int Hkv, qpk;             // key/value heads; query head h reads K/V head h / qpk
  int causal, window_left;  // window_left -1 = unlimited
  float scale;              // softmax scale
  float score_scale;        // scale * log2(e)
  int nkb;                  // key blocks per (batch, head)
  int nqb;                  // query blocks per (batch, head)
  unsigned long long wait_limit_ns;
  int* status;
  // dropout (DROP kernels): the forward's keep bits (keep_bits8 with these
  // values) and 1 / (1 - p)
  unsigned drop_threshold, seed_lo, seed_hi, drop_offset;
  float drop_scale;
};

template <int D>
struct BwdCfg {
  static constexpr int TILE = 128 * D * 2;        // one 128-row tile of 16-bit values
  static constexpr int NCHUNK = D / 64;           // 128-byte column chunks per row
  static constexpr int CHUNK = 128 * 128;         // one chunk of 128 rows
  static constexpr int HDR = 3072;                // barriers and the per-stage row statistics
  static constexpr int OFF_K = HDR;
  static constexpr int OFF_V = OFF_K + TILE;
  static constexpr int OFF_STAGE = OFF_V + TILE;  // 2 stages of (Q_i, dO_i)
  static constexpr int OFF_DS = OFF_STAGE + 2 * 2 * TILE;
  static constexpr int SMEM = OFF_DS + 128 * 128 * 2;
  static constexpr int S_COL = 0, P_COL = 64, DP_COL = 128;
  static constexpr int DV_COL = 256, DK_COL = 256 + D;
  static constexpr int DQ_COL = 256;             // dQ kernel
  static_assert(SMEM <= 232448, "shared memory budget");
  static_assert(D == 64 || D == 128, "head dim");
};

struct BwdHeader {
  uint64_t kv_full;
  uint64_t st_full[2], st_empty[2];   // (Q_i, dO_i) stages
  uint64_t s_full, dp_full;           // S^T, dP^T computed
  uint64_t p_ready;                   // P^T in TMEM
  uint64_t ds_ready;                  // dS^T in shared memory
  uint64_t ds_free;                   // the MMAs that read dS^T have completed
  uint64_t dkv_full;                  // every MMA of the CTA done
  uint32_t tmem_base;
  int abort_flag;
  float lse2[2][128];                 // LSE * log2(e) of the query block (+inf: row contributes nothing)
  float delta[2][128];
};
static_assert(sizeof(BwdHeader) <= 3072, "backward header");

constexpr int BWD_THREADS = 384;      // warpgroup 0: load + MMA; warps 4-11: gradients

__device__ __forceinline__ void bwd_error(BwdHeader* sh, const BwdParams& p, int code) {
  atomicOr(p.status, code);
  atomicExch(&sh->abort_flag, 1);
}

// Barrier 1 over the 256 gradient threads that also ANDs a flag across
// them, so every gradient warp takes the same exit decision.
__device__ __forceinline__ bool grad_bar_and(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 1, 256, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(v ? 1u : 0u)
      : "memory");
  return r != 0u;
}

// Query blocks that see key block jk: causal keeps queries at or after the
// key (absolute indices), a left window keeps queries at most window_left
// after it.
__device__ __forceinline__ void bwd_query_range(int jk, const BwdParams& p, int& i_lo, int& i_hi) {
  const int nqb = (p.Nq + 127) / 128;
  i_lo = p.causal ? jk : 0;
  i_hi = nqb - 1;
  if (p.window_left >= 0) {
    const long long last = static_cast<long long>(jk) * 128 + 127 + p.window_left;
    i_hi = static_cast<int>(min(static_cast<long long>(i_hi), last / 128));
  }
  if (jk * 128 >= p.Nk) i_hi = i_lo - 1;   // (not launched: the grid covers N_k)
}

template <int D, int DT, bool DROP>
__global__ void __launch_bounds__(BWD_THREADS, 1)
    fa_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                  const BwdParams p) {
  using C = BwdCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  if ((smem_u32(smem) & 1023u) != 0) {
    if (threadIdx.x == 0) atomicOr(p.status, ST_SMEM_MISALIGNED);
    return;
  }
  BwdHeader* sh = reinterpret_cast<BwdHeader*>(smem);
  const int warp = threadIdx.x / 32;
  // Head-major: the CTAs in flight are the key blocks of one or two heads,
  // so that head's Q, dO and dQ accumulator stay in L2 (longest first inside
  // a head: for causal attention key block 0 is seen by every query block).
  const int jk = static_cast<int>(blockIdx.x) % p.nkb;
  const int bhk = static_cast<int>(blockIdx.x) / p.nkb;   // (batch, K/V head)
  const int b = bhk / p.Hkv, hk = bhk - (bhk / p.Hkv) * p.Hkv;
  int i_lo, i_hi;
  bwd_query_range(jk, p, i_lo, i_hi);
  // The n-th query block a CTA visits is i_lo + (n + rot) mod cnt: causal
  // CTAs already start at their own diagonal; the others start at a block
  // of their own, so CTAs running side by side add into different dQ rows.
  const int cnt = i_hi - i_lo + 1;
  const int rot = (p.causal || cnt <= 0) ? 0 : jk % cnt;
  // every query head of the K/V head's group, cnt query blocks each: visit n
  // is query head hk * qpk + n / cnt, block i_lo + (n mod cnt + rot) mod cnt
  const int visits = cnt > 0 ? cnt * p.qpk : 0;
  const uint64_t lim = p.wait_limit_ns;

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&sh->kv_full), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(smem_u32(&sh->st_full[s]), 1);
      mbar_init(smem_u32(&sh->st_empty[s]), 1);
    }
    mbar_init(smem_u32(&sh->s_full), 1);
    mbar_init(smem_u32(&sh->dp_full), 1);
    mbar_init(smem_u32(&sh->p_ready), 256);
    mbar_init(smem_u32(&sh->ds_ready), 256);
    mbar_init(smem_u32(&sh->ds_free), 1);
    mbar_init(smem_u32(&sh->dkv_full), 1);
    sh->abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_map(&tm_q);
    tma_prefetch_map(&tm_k);
    tma_prefetch_map(&tm_v);
    tma_prefetch_map(&tm_do);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&sh->tmem_base), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = sh->tmem_base;
  const uint32_t sbase = smem_u32(smem);

  if (warp == 0) {
    // ---------------------------------------------------------- producer
    if (lane_id() == 0 && i_lo <= i_hi) {
      bool ok = true;
      const uint64_t pol_kv = policy_evict_first();
      const uint64_t pol_q = policy_evict_last();   // Q and dO blocks are read by many key blocks
      mbar_arrive_expect_tx(smem_u32(&sh->kv_full), 2 * C::TILE);
#pragma unroll
      for (int c = 0; c < C::NCHUNK; ++c) {
        tma_load_4d_hint(sbase + C::OFF_K + c * C::CHUNK, &tm_k, smem_u32(&sh->kv_full), c * 64, hk, jk * 128, b,
                         pol_kv);
        tma_load_4d_hint(sbase + C::OFF_V + c * C::CHUNK, &tm_v, smem_u32(&sh->kv_full), c * 64, hk, jk * 128, b,
                         pol_kv);
      }
      int n = 0;
      for (; n < visits; ++n) {
        const int hq = hk * p.qpk + n / cnt;
        const int i = i_lo + (n % cnt + rot) % cnt;
        const int s = n & 1;
        if (!mbar_wait(smem_u32(&sh->st_empty[s]), ((n >> 1) & 1) ^ 1, lim)) {
          bwd_error(sh, p, ST_TIMEOUT_LOAD);
          ok = false;
          break;
        }
        const uint32_t bar = smem_u32(&sh->st_full[s]);
        const uint32_t qdst = sbase + C::OFF_STAGE + s * 2 * C::TILE;
        mbar_arrive_expect_tx(bar, 2 * C::TILE);
#pragma unroll
        for (int c = 0; c < C::NCHUNK; ++c) {
          tma_load_4d_hint(qdst + c * C::CHUNK, &tm_q, bar, c * 64, hq, i * 128, b, pol_q);
          tma_load_4d_hint(qdst + C::TILE + c * C::CHUNK, &tm_do, bar, c * 64, hq, i * 128, b, pol_q);
        }
      }
      if (!ok) {
        // drain: the copies already issued land before the CTA exits
        mbar_wait(smem_u32(&sh->kv_full), 0, lim);
        for (int m = max(0, n - 2); m < n; ++m) mbar_wait(smem_u32(&sh->st_full[m & 1]), (m >> 1) & 1, lim);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane_id() == 0 && i_lo <= i_hi) {
      constexpr uint32_t FMT = DT == DT_BF16 ? 1u : 0u;
      constexpr uint32_t ID_ST = make_idesc(FMT, false, 128, 128);          // S^T, dP^T: both K-major
      constexpr uint32_t ID_KV = make_idesc(FMT, true, 128, D);             // dV, dK: A in TMEM, B M/N-major
      constexpr uint32_t HI = sdesc_sw128_hi(1024);
      const uint32_t k_kmaj = sdesc_sw128_lo(sbase + C::OFF_K, 16);
      const uint32_t v_kmaj = sdesc_sw128_lo(sbase + C::OFF_V, 16);
      const uint32_t ds_kmaj = sdesc_sw128_lo(sbase + C::OFF_DS, 16);
      // S^T = K Q_n^T for the n-th query block (keys on the lanes)
      auto issue_st = [&](int n) {
        const uint32_t q_kmaj = sdesc_sw128_lo(sbase + C::OFF_STAGE + (n & 1) * 2 * C::TILE, 16);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int byte = kk * 32;
          const uint32_t off = static_cast<uint32_t>(((byte / 128) * C::CHUNK + (byte % 128)) >> 4);
          mma_f16_ss_lo(tbase + C::S_COL, k_kmaj + off, q_kmaj + off, HI, ID_ST, kk > 0);
        }
        mma_commit(smem_u32(&sh->s_full));
      };
      // Per query block n: dP^T(n), then on P^T(n): dV(n) and the next
      // block's S^T (which overwrites S^T(n) under P^T(n), after dV(n) has
      // read it), then on dS^T(n): dK(n).  So dV(n) and S^T(n+1) run while
      // the gradient warps form dS, and dP^T(n+1) while they compute P(n+1).
      bool ok = mbar_wait(smem_u32(&sh->kv_full), 0, lim) && mbar_wait(smem_u32(&sh->st_full[0]), 0, lim);
      if (ok && visits > 0) {
        tc_fence_after();
        issue_st(0);
      }
      for (int n = 0; n < visits && ok; ++n) {
        const int s = n & 1;
        const uint32_t q_tile = sbase + C::OFF_STAGE + s * 2 * C::TILE;
        const uint32_t do_tile = q_tile + C::TILE;
        tc_fence_after();
        const uint32_t do_kmaj = sdesc_sw128_lo(do_tile, 16);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int byte = kk * 32;
          const uint32_t off = static_cast<uint32_t>(((byte / 128) * C::CHUNK + (byte % 128)) >> 4);
          mma_f16_ss_lo(tbase + C::DP_COL, v_kmaj + off, do_kmaj + off, HI, ID_ST, kk > 0);
        }
        mma_commit(smem_u32(&sh->dp_full));
        if (!mbar_wait(smem_u32(&sh->p_ready), n & 1, lim)) { ok = false; break; }
        tc_fence_after();
        // dV += P^T dO_n (A from TMEM: 16 queries = 8 columns per step)
        const uint32_t q_mn = sdesc_sw128_lo(q_tile, C::CHUNK), do_mn = sdesc_sw128_lo(do_tile, C::CHUNK);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = static_cast<uint32_t>((kk * 16 * 128) >> 4);
          mma_f16_ts_lo(tbase + C::DV_COL, tbase + C::P_COL + kk * 8, do_mn + off, HI, ID_KV, n > 0 || kk > 0);
        }
        if (n + 1 < visits) {
          if (!mbar_wait(smem_u32(&sh->st_full[(n + 1) & 1]), ((n + 1) >> 1) & 1, lim)) { ok = false; break; }
          tc_fence_after();
          issue_st(n + 1);
        }
        if (!mbar_wait(smem_u32(&sh->ds_ready), n & 1, lim)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          // dK += dS^T Q_n: A = dS^T in shared memory, K-major (16 queries = 32 bytes of a row)
          const int byte = kk * 32;
          const uint32_t a_off = static_cast<uint32_t>(((byte / 128) * C::CHUNK + (byte % 128)) >> 4);
          const uint32_t b_off = static_cast<uint32_t>((kk * 16 * 128) >> 4);
          mma_f16_ss_lo(tbase + C::DK_COL, ds_kmaj + a_off, q_mn + b_off, HI, ID_KV, n > 0 || kk > 0);
        }
        mma_commit(smem_u32(&sh->st_empty[s]));   // last readers of Q_n and dO_n
        mma_commit(smem_u32(&sh->ds_free));       // ... and of dS^T(n)
      }
      if (!ok) bwd_error(sh, p, ST_TIMEOUT_MMA);
      mma_commit(smem_u32(&sh->dkv_full));   // also: every MMA done before TMEM is released
      if (!ok) mbar_wait(smem_u32(&sh->dkv_full), 0, lim);
    }
  } else if (warp >= 4) {
    // ---------------------------------------------------------- gradients
    const int quad = warp & 3;
    const int sub = (warp - 4) >> 2;
    const int lane = static_cast<int>(lane_id());
    const int half = lane >> 4;
    const int r = quad * 32 + sub * 16 + (lane & 15);           // TMEM lane: key (S^T, dK, dV) or query (dQ)
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32 + sub * 16) << 16;
    const int t = static_cast<int>(threadIdx.x) - 128;          // 0..255
    const int key = jk * 128 + r;
    const float c2 = p.score_scale;
    uint8_t* ds_row = smem + C::OFF_DS + half * C::CHUNK + r * 128;
    bool ok = true;
    bool dq_ok = true;   // this block's later waits (reported at the next vote)
    for (int n = 0; n < visits; ++n) {
      const int hq = hk * p.qpk + n / cnt;
      const int i = i_lo + (n % cnt + rot) % cnt;
      const long long bhq = (static_cast<long long>(b) * p.H + hq) * p.Nq;
      const int buf = n & 1;
      // row statistics of query block i (one value per thread); the vote
      // below is also the barrier that publishes them
      {
        const int q = i * 128 + (t & 127);
        if (t < 128) {
          float v = INFINITY;   // rows past N_q or without a visible key contribute nothing
          if (q < p.Nq) {
            const float l = p.lse[bhq + q];
            if (l != -INFINITY) v = l * 1.4426950408889634f;
          }
          sh->lse2[buf][t] = v;
        } else {
          sh->delta[buf][t - 128] = q < p.Nq ? p.delta[bhq + q] : 0.f;
        }
      }
      const int q0 = i * 128;
      const bool need_mask = (jk * 128 + 128 > p.Nk) || (p.causal && jk * 128 + 127 > q0) ||
                             (p.window_left >= 0 && jk * 128 < q0 + 127 - p.window_left);
      const bool got = mbar_wait(smem_u32(&sh->s_full), n & 1, lim);
      if (!grad_bar_and(got && dq_ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
      // the thread's half row of S^T (queries half * 64 + [0, 64)) in
      // registers before any P^T store lands over its upper half
      float pv[64];
      tmem_ld_16x32bx2_x32<64>(tbase + lane_off + C::S_COL, reinterpret_cast<uint32_t*>(pv));
      tmem_ld_16x32bx2_x32<64>(tbase + lane_off + C::S_COL + 32, reinterpret_cast<uint32_t*>(pv + 32));
      tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 64; ++e) {
        const int ql = half * 64 + e;
        float pe = ex2_approx(pv[e] * c2 - sh->lse2[buf][ql]);
        if (need_mask) {
          const int q = q0 + ql;
          const bool vis = key < p.Nk && (!p.causal || key <= q) && (p.window_left < 0 || key >= q - p.window_left);
          pe = vis ? pe : 0.f;
        }
        pv[e] = pe;
      }
      // dropout keep bits of this thread's key for its 64 queries (bit e:
      // query q0 + 64 * half + e).  The generator gives 8 keys of one query
      // per call, so in round m lane L draws query 8m + (L mod 8) for its
      // 8-key group, and the 8 lanes of the group exchange bits
      uint32_t keep[2] = {0u, 0u};
      if constexpr (DROP) {
        const int lane8 = lane & 7;
        const uint32_t grp = static_cast<uint32_t>(jk * 128 + quad * 32 + sub * 16 + (lane & 8)) / 8u;
        const uint32_t bh = static_cast<uint32_t>(b * p.H + hq);
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          const uint32_t qq = static_cast<uint32_t>(q0 + half * 64 + 8 * m + lane8);
          const uint32_t mine8 = keep_bits8(grp, qq, bh, p.drop_offset, p.seed_lo, p.seed_hi, p.drop_threshold);
          uint32_t got8 = 0;
#pragma unroll
          for (int x = 0; x < 8; ++x) {
            const uint32_t v8 = __shfl_sync(0xffffffffu, mine8, (lane & ~7) + x);
            got8 |= ((v8 >> lane8) & 1u) << x;
          }
          keep[m / 4] |= got8 << (8 * (m % 4));
        }
      }
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t pw[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          float p0 = pv[c * 32 + 2 * e], p1 = pv[c * 32 + 2 * e + 1];
          if constexpr (DROP) {
            // dV takes the kept probabilities, scaled by 1 / (1 - p)
            const uint32_t kb = keep[c] >> (2 * e);
            p0 = (kb & 1u) ? p0 * p.drop_scale : 0.f;
            p1 = (kb & 2u) ? p1 * p.drop_scale : 0.f;
          }
          pw[e] = pack2<DT>(p0, p1);
        }
        tmem_st_16x32bx2_x16<32>(tbase + lane_off + C::P_COL + c * 16, pw);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(smem_u32(&sh->p_ready));
      // dP^T(n) (committed after S^T(n); a wait that times out leaves dS
      // unusable, which the next vote reports)
      dq_ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&sh->dp_full), n & 1, lim)) && dq_ok;
      // dS^T(n - 1) in shared memory has been read by dK(n - 1)
      if (n > 0) dq_ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&sh->ds_free), (n - 1) & 1, lim)) && dq_ok;
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        // dS^T for queries half * 64 + [16c, 16c + 16)
        uint32_t dpv[16];
        tmem_ld_16x32bx2_x16<64>(tbase + lane_off + C::DP_COL + c * 16, dpv);
        tmem_wait_ld();
        uint32_t dw[8];
#pragma unroll
        for (int e = 0; e < 16; e += 2) {
          const int ql = half * 64 + c * 16 + e;
          float g0 = __uint_as_float(dpv[e]), g1 = __uint_as_float(dpv[e + 1]);
          if constexpr (DROP) {
            // dP of the dropped forward: Z / (1 - p) times dO V^T
            const uint32_t kb = keep[(c * 16 + e) / 32] >> ((c * 16 + e) % 32);
            g0 = (kb & 1u) ? g0 * p.drop_scale : 0.f;
            g1 = (kb & 2u) ? g1 * p.drop_scale : 0.f;
          }
          const float d0 = pv[c * 16 + e] * (g0 - sh->delta[buf][ql]);
          const float d1 = pv[c * 16 + e + 1] * (g1 - sh->delta[buf][ql + 1]);
          dw[e / 2] = pack2<DT>(d0, d1);
        }
        // row r of dS^T, two 16-byte units of the 128-byte row, XOR-swizzled
        // by (r mod 8) like a TMA 128B tile
        const int u0 = (2 * c) ^ (r & 7), u1 = (2 * c + 1) ^ (r & 7);
        *reinterpret_cast<uint4*>(ds_row + u0 * 16) = make_uint4(dw[0], dw[1], dw[2], dw[3]);
        *reinterpret_cast<uint4*>(ds_row + u1 * 16) = make_uint4(dw[4], dw[5], dw[6], dw[7]);
      }
      fence_proxy_async_smem();   // dS^T stores visible to the MMA's reads
      tc_fence_before();
      mbar_arrive(smem_u32(&sh->ds_ready));
    }
    if (!grad_bar_and(ok && dq_ok)) {
      ok = false;
      if (threadIdx.x == 128) bwd_error(sh, p, ST_TIMEOUT_SOFTMAX);
    }
    // dK, dV of this key block (zero when no query sees it)
    const bool have = i_lo <= i_hi;
    if (ok && have) {
      bool got = mbar_wait(smem_u32(&sh->dkv_full), 0, lim);
      got = __all_sync(0xffffffffu, got);
      if (!got) { bwd_error(sh, p, ST_TIMEOUT_SOFTMAX); ok = false; }
      tc_fence_after();
    }
    if (ok) {
      const long long row = (static_cast<long long>(b) * p.Nk + key) * p.Hkv + hk;
      uint8_t* dv_row = reinterpret_cast<uint8_t*>(p.dv) + (row * D + half * (D / 2)) * 2;
      uint8_t* dk_row = reinterpret_cast<uint8_t*>(p.dk) + (row * D + half * (D / 2)) * 2;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t v[16], k[16];
        if (have) {
          tmem_ld_16x32bx2_x16<D / 2>(tbase + lane_off + C::DV_COL + c * 16, v);
          tmem_ld_16x32bx2_x16<D / 2>(tbase + lane_off + C::DK_COL + c * 16, k);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int e = 0; e < 16; ++e) v[e] = k[e] = 0u;
        }
        if (key < p.Nk) {
          store_out_row16<DT>(dv_row + c * 32, reinterpret_cast<const float*>(v), 1.f);
          store_out_row16<DT>(dk_row + c * 32, reinterpret_cast<const float*>(k), p.scale);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

// dQ kernel: one CTA per (batch, head, 128-query block i), head-major, the
// query blocks with the most keys first.  Warp 0 loads Q_i and dO_i once and
// K_j, V_j of every key block the queries see through two stages; warp 1
// issues S = Q_i K_j^T and dP = dO_i V_j^T (queries on the lanes), then on
// dS(j): dQ += dS K_j (A = dS from TMEM), then the next block's S and dP at
// once; warps 4-11 form dS = P * (dP - D) with P = exp(S - LSE).
struct DqHeader {
  uint64_t q_full;
  uint64_t kv_full[2], kv_empty[2];
  uint64_t dp_full;          // S(j) and dP(j) computed
  uint64_t ds_ready;         // dS(j) in TMEM
  uint64_t dq_done;          // every MMA done
  uint32_t tmem_base;
  int abort_flag;
};

template <int D, int DT, bool DROP>
__global__ void __launch_bounds__(BWD_THREADS, 1)
    fa_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                     const BwdParams p) {
  using C = BwdCfg<D>;
  constexpr int OFF_Q = 1024, OFF_DO = OFF_Q + C::TILE, OFF_KV = OFF_DO + C::TILE;   // then 2 x (K, V)
  extern __shared__ __align__(1024) uint8_t smem[];
  if ((smem_u32(smem) & 1023u) != 0) {
    if (threadIdx.x == 0) atomicOr(p.status, ST_SMEM_MISALIGNED);
    return;
  }
  DqHeader* sh = reinterpret_cast<DqHeader*>(smem);
  const int warp = threadIdx.x / 32;
  const int iq = p.nqb - 1 - static_cast<int>(blockIdx.x) % p.nqb;
  const int bh = static_cast<int>(blockIdx.x) / p.nqb;
  const int b = bh / p.H, h = bh - (bh / p.H) * p.H;
  const int hk = h / p.qpk;   // this query head's K/V head
  const int q0 = iq * 128;
  // key blocks the rows of this query block see (as in the forward)
  const int qe = min(q0 + 127, p.Nq - 1);
  const int j_lo = p.window_left >= 0 ? max(0, q0 - p.window_left) / 128 : 0;
  const int j_hi = p.causal ? min(qe, p.Nk - 1) / 128 : p.nkb - 1;
  const int cnt = (q0 < p.Nq && p.Nk > 0) ? max(0, j_hi - j_lo + 1) : 0;
  const uint64_t lim = p.wait_limit_ns;

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&sh->q_full), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(smem_u32(&sh->kv_full[s]), 1);
      mbar_init(smem_u32(&sh->kv_empty[s]), 1);
    }
    mbar_init(smem_u32(&sh->dp_full), 1);
    mbar_init(smem_u32(&sh->ds_ready), 256);
    mbar_init(smem_u32(&sh->dq_done), 1);
    sh->abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_map(&tm_q);
    tma_prefetch_map(&tm_k);
    tma_prefetch_map(&tm_v);
    tma_prefetch_map(&tm_do);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&sh->tmem_base), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = sh->tmem_base;
  const uint32_t sbase = smem_u32(smem);

  if (warp == 0) {
    if (lane_id() == 0 && cnt > 0) {
      bool ok = true;
      const uint64_t pol_q = policy_evict_first();
      const uint64_t pol_kv = policy_evict_last();   // K, V of a head are read by all its query blocks
      mbar_arrive_expect_tx(smem_u32(&sh->q_full), 2 * C::TILE);
#pragma unroll
      for (int c = 0; c < C::NCHUNK; ++c) {
        tma_load_4d_hint(sbase + OFF_Q + c * C::CHUNK, &tm_q, smem_u32(&sh->q_full), c * 64, h, q0, b, pol_q);
        tma_load_4d_hint(sbase + OFF_DO + c * C::CHUNK, &tm_do, smem_u32(&sh->q_full), c * 64, h, q0, b, pol_q);
      }
      int n = 0;
      for (; n < cnt; ++n) {
        const int j = j_lo + n, s = n & 1;
        if (!mbar_wait(smem_u32(&sh->kv_empty[s]), ((n >> 1) & 1) ^ 1, lim)) {
          atomicOr(p.status, ST_TIMEOUT_LOAD);
          ok = false;
          break;
        }
        const uint32_t bar = smem_u32(&sh->kv_full[s]);
        const uint32_t kdst = sbase + OFF_KV + s * 2 * C::TILE;
        mbar_arrive_expect_tx(bar, 2 * C::TILE);
#pragma unroll
        for (int c = 0; c < C::NCHUNK; ++c) {
          tma_load_4d_hint(kdst + c * C::CHUNK, &tm_k, bar, c * 64, hk, j * 128, b, pol_kv);
          tma_load_4d_hint(kdst + C::TILE + c * C::CHUNK, &tm_v, bar, c * 64, hk, j * 128, b, pol_kv);
        }
      }
      if (!ok) {
        mbar_wait(smem_u32(&sh->q_full), 0, lim);
        for (int m = max(0, n - 2); m < n; ++m) mbar_wait(smem_u32(&sh->kv_full[m & 1]), (m >> 1) & 1, lim);
      }
    }
  } else if (warp == 1) {
    if (lane_id() == 0 && cnt > 0) {
      constexpr uint32_t FMT = DT == DT_BF16 ? 1u : 0u;
      constexpr uint32_t ID_S = make_idesc(FMT, false, 128, 128);   // S, dP: both K-major
      constexpr uint32_t ID_Q = make_idesc(FMT, true, 128, D);      // dQ: A in TMEM, B head-dim-major
      constexpr uint32_t HI = sdesc_sw128_hi(1024);
      const uint32_t q_kmaj = sdesc_sw128_lo(sbase + OFF_Q, 16);
      const uint32_t do_kmaj = sdesc_sw128_lo(sbase + OFF_DO, 16);
      // S(n) and dP(n) for the n-th key block
      auto issue_s_dp = [&](int n) {
        const uint32_t kt = sbase + OFF_KV + (n & 1) * 2 * C::TILE;
        const uint32_t k_kmaj = sdesc_sw128_lo(kt, 16), v_kmaj = sdesc_sw128_lo(kt + C::TILE, 16);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int byte = kk * 32;
          const uint32_t off = static_cast<uint32_t>(((byte / 128) * C::CHUNK + (byte % 128)) >> 4);
          mma_f16_ss_lo(tbase + C::S_COL, q_kmaj + off, k_kmaj + off, HI, ID_S, kk > 0);
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int byte = kk * 32;
          const uint32_t off = static_cast<uint32_t>(((byte / 128) * C::CHUNK + (byte % 128)) >> 4);
          mma_f16_ss_lo(tbase + C::DP_COL, do_kmaj + off, v_kmaj + off, HI, ID_S, kk > 0);
        }
        mma_commit(smem_u32(&sh->dp_full));
      };
      bool ok = mbar_wait(smem_u32(&sh->q_full), 0, lim) && mbar_wait(smem_u32(&sh->kv_full[0]), 0, lim);
      if (ok) {
        tc_fence_after();
        issue_s_dp(0);
      }
      for (int n = 0; n < cnt && ok; ++n) {
        if (!mbar_wait(smem_u32(&sh->ds_ready), n & 1, lim)) { ok = false; break; }
        tc_fence_after();
        // dQ += dS K_n: A = dS (16-bit, over S's upper half), 16 keys = 8 columns per step
        const uint32_t k_mn = sdesc_sw128_lo(sbase + OFF_KV + (n & 1) * 2 * C::TILE, C::CHUNK);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = static_cast<uint32_t>((kk * 16 * 128) >> 4);
          mma_f16_ts_lo(tbase + C::DQ_COL, tbase + C::P_COL + kk * 8, k_mn + off, HI, ID_Q, n > 0 || kk > 0);
        }
        mma_commit(smem_u32(&sh->kv_empty[n & 1]));   // last readers of K_n, V_n
        if (n + 1 < cnt) {
          // S(n+1) overwrites dS(n) after dQ(n) has read it (same pipe, in order)
          if (!mbar_wait(smem_u32(&sh->kv_full[(n + 1) & 1]), ((n + 1) >> 1) & 1, lim)) { ok = false; break; }
          tc_fence_after();
          issue_s_dp(n + 1);
        }
      }
      if (!ok) atomicOr(p.status, ST_TIMEOUT_MMA);
      mma_commit(smem_u32(&sh->dq_done));
      if (!ok) mbar_wait(smem_u32(&sh->dq_done), 0, lim);
    }
  } else if (warp >= 4) {
    const int quad = warp & 3;
    const int sub = (warp - 4) >> 2;
    const int lane = static_cast<int>(lane_id());
    const int half = lane >> 4;
    const int r = quad * 32 + sub * 16 + (lane & 15);        // TMEM lane: query row
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32 + sub * 16) << 16;
    const int q = q0 + r;
    const long long bhq = static_cast<long long>(bh) * p.Nq;
    // this row's statistics: LSE * log2(e) (+inf: the row contributes nothing) and D
    float lse2 = INFINITY, dlt = 0.f;
    if (q < p.Nq) {
      const float l = p.lse[bhq + q];
      if (l != -INFINITY) lse2 = l * 1.4426950408889634f;
      dlt = p.delta[bhq + q];
    }
    const float c2 = p.score_scale;
    bool ok = true;
    for (int n = 0; n < cnt; ++n) {
      const int k0 = (j_lo + n) * 128;
      const bool need_mask = (k0 + 128 > p.Nk) || (p.causal && k0 + 127 > q0) ||
                             (p.window_left >= 0 && k0 < q0 + 127 - p.window_left);
      if (!grad_bar_and(mbar_wait(smem_u32(&sh->dp_full), n & 1, lim))) {
        ok = false;
        break;
      }
      // dropout keep bits of this row's keys k0 + 64 * half + [0, 64)
      uint32_t keep[2] = {0u, 0u};
      if constexpr (DROP) {
        const uint32_t g0 = static_cast<uint32_t>(k0 + half * 64) / 8u;
        const uint32_t bhq = static_cast<uint32_t>(b * p.H + h);
#pragma unroll
        for (int g = 0; g < 8; ++g)
          keep[g / 4] |= keep_bits8(g0 + g, static_cast<uint32_t>(q), bhq, p.drop_offset, p.seed_lo, p.seed_hi,
                                    p.drop_threshold)
                         << (8 * (g % 4));
      }
      tc_fence_after();
      // the whole half row of S (keys half * 64 + [0, 64)) before any dS store
      float pv[64];
      tmem_ld_16x32bx2_x32<64>(tbase + lane_off + C::S_COL, reinterpret_cast<uint32_t*>(pv));
      tmem_ld_16x32bx2_x32<64>(tbase + lane_off + C::S_COL + 32, reinterpret_cast<uint32_t*>(pv + 32));
      tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 64; ++e) {
        float pe = ex2_approx(pv[e] * c2 - lse2);
        if (need_mask) {
          const int key = k0 + half * 64 + e;
          const bool vis = key < p.Nk && (!p.causal || key <= q) && (p.window_left < 0 || key >= q - p.window_left);
          pe = vis ? pe : 0.f;
        }
        pv[e] = pe;
      }
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t dpv[16];
        tmem_ld_16x32bx2_x16<64>(tbase + lane_off + C::DP_COL + c * 16, dpv);
        tmem_wait_ld();
        uint32_t dw[8];
#pragma unroll
        for (int e = 0; e < 16; e += 2) {
          float g0 = __uint_as_float(dpv[e]), g1 = __uint_as_float(dpv[e + 1]);
          if constexpr (DROP) {
            // dP of the dropped forward: Z / (1 - p) times dO V^T
            const uint32_t kb = keep[(c * 16 + e) / 32] >> ((c * 16 + e) % 32);
            g0 = (kb & 1u) ? g0 * p.drop_scale : 0.f;
            g1 = (kb & 2u) ? g1 * p.drop_scale : 0.f;
          }
          dw[e / 2] = pack2<DT>(pv[c * 16 + e] * (g0 - dlt), pv[c * 16 + e + 1] * (g1 - dlt));
        }
        tmem_st_16x32bx2_x8<32>(tbase + lane_off + C::P_COL + c * 8, dw);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(smem_u32(&sh->ds_ready));
    }
    if (!ok && threadIdx.x == 128) atomicOr(p.status, ST_TIMEOUT_SOFTMAX);
    // dQ = scale * (sum over key blocks of dS K), 16-bit
    bool have = ok && cnt > 0;
    if (have) {
      have = __all_sync(0xffffffffu, mbar_wait(smem_u32(&sh->dq_done), 0, lim));
      if (!have && lane == 0) atomicOr(p.status, ST_TIMEOUT_SOFTMAX);
      tc_fence_after();
    }
    // (the TMEM loads are warp-collective: every lane takes them, whatever
    // its row; only rows inside N_q are stored)
    if (have || cnt == 0) {
      uint8_t* dq_row = reinterpret_cast<uint8_t*>(p.dq) +
                        (((static_cast<long long>(b) * p.Nq + q) * p.H + h) * D + half * (D / 2)) * 2;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t v[16];
        if (cnt > 0) {
          tmem_ld_16x32bx2_x16<D / 2>(tbase + lane_off + C::DQ_COL + c * 16, v);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int e = 0; e < 16; ++e) v[e] = 0u;
        }
        if (q < p.Nq) store_out_row16<DT>(dq_row + c * 32, reinterpret_cast<const float*>(v), p.scale);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

// D_i = sum_d dO_id O_id (fp32) for every (b, h, i).  One warp per (b, i, h)
// row.
template <int D>
__global__ void fa_bwd_prologue_kernel(const void* __restrict__ out, const void* __restrict__ dout, int dt,
                                       float* __restrict__ delta, int B, int Nq, int H) {
  constexpr int PER = D / 32;
  const long long rows = static_cast<long long>(B) * Nq * H;
  const int lane = static_cast<int>(threadIdx.x & 31u);
  const long long warps = static_cast<long long>(gridDim.x) * (blockDim.x / 32);
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x / 32) + threadIdx.x / 32; i < rows; i += warps) {
    float acc = 0.f;
    const long long base = i * D + lane * PER;
#pragma unroll
    for (int e = 0; e < PER; ++e) {
      float o, g;
      if (dt == DT_BF16) {
        o = __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(out)[base + e]);
        g = __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(dout)[base + e]);
      } else {
        o = __half2float(reinterpret_cast<const __half*>(out)[base + e]);
        g = __half2float(reinterpret_cast<const __half*>(dout)[base + e]);
      }
      acc = fmaf(o, g, acc);
    }
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, m);
    if (lane == 0) {
      // i enumerates (b, n, h); D_i is stored [B, H, N_q] like the LSE
      const long long h = i % H, bn = i / H, nq = bn % Nq, bb = bn / Nq;
      delta[(bb * H + h) * Nq + nq] = acc;
    }
  }
}

}  // namespace fa
