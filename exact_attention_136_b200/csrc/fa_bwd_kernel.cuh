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
// One CTA per (batch, head, 128-key block): K_j and V_j stay in shared
// memory and dK_j, dV_j accumulate in tensor memory over the query blocks
// that see the keys; dQ is a sum over key blocks, so every CTA adds its
// share into an fp32 buffer: the gradient warps stage it through shared
// memory in 128-byte lines and the TMA adds the boxes into global memory
// (cp.reduce.async.bulk.tensor .add).
//
// Everything is computed transposed (keys on the TMEM lanes).  P^T, written
// back into tensor memory over S^T by the gradient warps (after each has
// read its whole half row of S^T), is the A operand of dV += P^T dO.  dS^T
// goes to shared memory in the 128-byte-swizzled layout, where the MMA reads
// it both ways: K-major for dK += dS^T Q and M-major (queries contiguous) as
// the dS of dQ = dS K.
//
// Tensor memory (512 columns): S^T [0,128) with P^T (16-bit) over its upper
// half [64,128), dP^T [128,256), dV [256,256+D), dK [256+D,256+2D).  dQ
// (queries x D) goes to [384,448) for D = 64; for D = 128 there is no room
// left, so it takes dP^T's columns (dead once the gradient warps have read
// them) and the next dP^T waits until the gradient warps have read dQ out.
#pragma once

namespace fa {

struct BwdParams {
  void* dk;                 // [B, N_k, H, D], 16-bit like the inputs
  void* dv;                 // [B, N_k, H, D]
  float* dq_acc;            // [B, N_q, H, D] fp32, zero on entry; receives scale * dS K
  const float* lse;         // [B, H, N_q] natural log (forward output)
  const float* delta;       // [B, H, N_q] rowsum(dO * O)
  int B, Nq, Nk, H;
  int causal, window_left;  // window_left -1 = unlimited
  float scale;              // softmax scale
  float score_scale;        // scale * log2(e)
  int nkb;                  // key blocks per (batch, head)
  unsigned long long wait_limit_ns;
  int* status;
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
  static constexpr bool SERIAL_DQ = D == 128;
  static constexpr int DQ_COL = SERIAL_DQ ? DP_COL : 256 + 2 * D;
  static_assert(SMEM <= 232448, "shared memory budget");
  static_assert(D == 64 || D == 128, "head dim");
};

struct BwdHeader {
  uint64_t kv_full;
  uint64_t st_full[2], st_empty[2];   // (Q_i, dO_i) stages
  uint64_t s_full, dp_full;           // S^T, dP^T computed
  uint64_t p_ready;                   // P^T in TMEM
  uint64_t ds_ready;                  // dS^T in shared memory
  uint64_t dq_full, dq_empty;         // dQ partial computed / read out
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

// Bulk tensor reduce-add (TMA) of a shared-memory box into global memory,
// and the bulk-group bookkeeping around it.
__device__ __forceinline__ void tma_reduce_add_4d(const CUtensorMap* map, uint32_t src, int c0, int c1, int c2,
                                                  int c3) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.4d.global.shared::cta.add.tile.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(
          map),
      "r"(src), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}
__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// the shared-memory sources of every committed bulk operation have been read
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// ... and the operations have completed
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

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

template <int D, int DT>
__global__ void __launch_bounds__(BWD_THREADS, 1)
    fa_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                  const __grid_constant__ CUtensorMap tm_dq, const BwdParams p) {
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
  const int bh = static_cast<int>(blockIdx.x) / p.nkb;
  const int b = bh / p.H, h = bh - (bh / p.H) * p.H;
  int i_lo, i_hi;
  bwd_query_range(jk, p, i_lo, i_hi);
  // The n-th query block a CTA visits is i_lo + (n + rot) mod cnt: causal
  // CTAs already start at their own diagonal; the others start at a block
  // of their own, so CTAs running side by side add into different dQ rows.
  const int cnt = i_hi - i_lo + 1;
  const int rot = (p.causal || cnt <= 0) ? 0 : jk % cnt;
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
    mbar_init(smem_u32(&sh->dq_full), 1);
    mbar_init(smem_u32(&sh->dq_empty), 256);
    mbar_init(smem_u32(&sh->dkv_full), 1);
    sh->abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_map(&tm_q);
    tma_prefetch_map(&tm_k);
    tma_prefetch_map(&tm_v);
    tma_prefetch_map(&tm_do);
    tma_prefetch_map(&tm_dq);
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
        tma_load_4d_hint(sbase + C::OFF_K + c * C::CHUNK, &tm_k, smem_u32(&sh->kv_full), c * 64, h, jk * 128, b,
                         pol_kv);
        tma_load_4d_hint(sbase + C::OFF_V + c * C::CHUNK, &tm_v, smem_u32(&sh->kv_full), c * 64, h, jk * 128, b,
                         pol_kv);
      }
      int n = 0;
      for (; n < cnt; ++n) {
        const int i = i_lo + (n + rot) % cnt;
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
          tma_load_4d_hint(qdst + c * C::CHUNK, &tm_q, bar, c * 64, h, i * 128, b, pol_q);
          tma_load_4d_hint(qdst + C::TILE + c * C::CHUNK, &tm_do, bar, c * 64, h, i * 128, b, pol_q);
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
      constexpr uint32_t ID_Q = make_idesc(FMT, true, 128, D) | (1u << 15); // dQ: A and B M/N-major
      constexpr uint32_t HI = sdesc_sw128_hi(1024);
      const uint32_t k_kmaj = sdesc_sw128_lo(sbase + C::OFF_K, 16);
      const uint32_t v_kmaj = sdesc_sw128_lo(sbase + C::OFF_V, 16);
      const uint32_t k_mn = sdesc_sw128_lo(sbase + C::OFF_K, C::CHUNK);
      const uint32_t ds_mn = sdesc_sw128_lo(sbase + C::OFF_DS, C::CHUNK);
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
      // read it), then on dS^T(n): dK(n) and dQ(n).  So dV(n) and S^T(n+1)
      // run while the gradient warps form dS, and dP^T(n+1) while they
      // compute P(n+1).
      bool ok = mbar_wait(smem_u32(&sh->kv_full), 0, lim) && mbar_wait(smem_u32(&sh->st_full[0]), 0, lim);
      if (ok) {
        tc_fence_after();
        issue_st(0);
      }
      for (int n = 0; n < cnt && ok; ++n) {
        const int s = n & 1;
        const uint32_t q_tile = sbase + C::OFF_STAGE + s * 2 * C::TILE;
        const uint32_t do_tile = q_tile + C::TILE;
        // (D = 128: dP^T's columns hold the previous block's dQ until it is read out)
        if (C::SERIAL_DQ && n > 0 && !mbar_wait(smem_u32(&sh->dq_empty), (n - 1) & 1, lim)) {
          ok = false;
          break;
        }
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
        if (n + 1 < cnt) {
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
        // dQ_n (partial) = dS K_j: A = dS^T read query-major, B = K_j head-dim-major
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = static_cast<uint32_t>((kk * 16 * 128) >> 4);
          mma_f16_ss_lo(tbase + C::DQ_COL, ds_mn + off, k_mn + off, HI, ID_Q, kk > 0);
        }
        mma_commit(smem_u32(&sh->dq_full));
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
    const long long bhq = static_cast<long long>(bh) * p.Nq;
    bool ok = true;
    bool dq_ok = true;   // the previous block's dQ wait (reported at the next vote)
    for (int n = 0; n < cnt; ++n) {
      const int i = i_lo + (n + rot) % cnt;
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
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t pw[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) pw[e] = pack2<DT>(pv[c * 32 + 2 * e], pv[c * 32 + 2 * e + 1]);
        tmem_st_16x32bx2_x16<32>(tbase + lane_off + C::P_COL + c * 16, pw);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(smem_u32(&sh->p_ready));
      // dP^T(n) (committed after S^T(n); a wait that times out leaves dS
      // unusable, which the next vote reports)
      dq_ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&sh->dp_full), n & 1, lim)) && dq_ok;
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
          const float d0 = pv[c * 16 + e] * (__uint_as_float(dpv[e]) - sh->delta[buf][ql]);
          const float d1 = pv[c * 16 + e + 1] * (__uint_as_float(dpv[e + 1]) - sh->delta[buf][ql + 1]);
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
      // dQ_i partial (queries on the lanes), staged as scale * dQ through the
      // dS buffer (its readers, the dK and dQ MMAs, have completed) in boxes
      // of 32 columns x 128 rows, 128-byte swizzled, and added into dq_acc by
      // the TMA; rows past N_q are clipped by the map.  Thread (r, half)
      // holds columns half * D/2 + [0, D/2): round k stages columns
      // half * D/2 + 32k + [0, 32) as box `half`.  The TMEM columns are
      // released once the last round's values are in registers.
      dq_ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&sh->dq_full), n & 1, lim)) && dq_ok;
      tc_fence_after();
#pragma unroll
      for (int k = 0; k < D / 64; ++k) {
        uint8_t* box_row = smem + C::OFF_DS + half * (32 * 128 * 4) + r * 128;
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          float dqv[16];
          if (dq_ok) {
            tmem_ld_16x32bx2_x16<D / 2>(tbase + lane_off + C::DQ_COL + 32 * k + 16 * cc,
                                        reinterpret_cast<uint32_t*>(dqv));
            tmem_wait_ld();
          }
#pragma unroll
          for (int u = 0; u < 4; ++u)
            *reinterpret_cast<float4*>(box_row + (((4 * cc + u) ^ (r & 7)) * 16)) =
                make_float4(p.scale * dqv[4 * u], p.scale * dqv[4 * u + 1], p.scale * dqv[4 * u + 2],
                            p.scale * dqv[4 * u + 3]);
        }
        if (k == D / 64 - 1) {
          tc_fence_before();
          mbar_arrive(smem_u32(&sh->dq_empty));
        }
        fence_proxy_async_smem();
        asm volatile("bar.sync 1, 256;" ::: "memory");
        if (t == 0) {
#pragma unroll
          for (int hb = 0; hb < 2; ++hb)
            tma_reduce_add_4d(&tm_dq, sbase + C::OFF_DS + hb * (32 * 128 * 4), hb * (D / 2) + 32 * k, h, q0, b);
          bulk_commit_group();
          bulk_wait_read_all();   // the buffer may be written again
        }
        asm volatile("bar.sync 1, 256;" ::: "memory");
      }
    }
    if (t == 0) bulk_wait_all();   // every reduction has landed before the CTA exits
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
      const long long row = (static_cast<long long>(b) * p.Nk + key) * p.H + h;
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

// D_i = sum_d dO_id O_id (fp32) for every (b, h, i), and dq_acc = 0.  One warp
// per (b, i, h) row.
template <int D>
__global__ void fa_bwd_prologue_kernel(const void* __restrict__ out, const void* __restrict__ dout, int dt,
                                       float* __restrict__ delta, float* __restrict__ dq_acc, int B, int Nq,
                                       int H) {
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
      dq_acc[base + e] = 0.f;
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

// dQ = dq_acc converted to the input's 16-bit type.
__global__ void fa_bwd_epilogue_kernel(const float* __restrict__ dq_acc, void* dq, int dt, long long n) {
  for (long long i = (blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x) * 4; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x * 4) {
    const float4 v = *reinterpret_cast<const float4*>(dq_acc + i);
    uint2 w;
    if (dt == DT_BF16) {
      w.x = pack2<DT_BF16>(v.x, v.y);
      w.y = pack2<DT_BF16>(v.z, v.w);
    } else {
      w.x = pack2<DT_FP16>(v.x, v.y);
      w.y = pack2<DT_FP16>(v.z, v.w);
    }
    *reinterpret_cast<uint2*>(reinterpret_cast<uint8_t*>(dq) + i * 2) = w;
  }
}

}  // namespace fa
