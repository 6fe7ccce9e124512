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
// P^T goes to shared memory in the 128-byte-swizzled layout, read K-major as
// the A operand of dV += P^T dO; dS^T, written back into tensor memory over
// the upper half of dP^T by the gradient warps (after each warp has read all
// of its dP^T), is the A operand of dK += dS^T Q.  S^T is released as soon as
// the gradient warps hold it in registers, so the next block's S^T is
// computed while they form P and dS.  Tensor memory: S^T [0,128),
// dP^T [128,256) with dS^T (16-bit) over [192,256), dV [256,256+D),
// dK [256+D,256+2D).
//
// dQ kernel: queries on the lanes, like the forward: S [0,128), dP [128,256),
// dS (16-bit) written over S's upper half [64,128) as the A operand of
// dQ += dS K, dQ [256,256+D).
#pragma once

namespace fa {

// Timeline records of CTA 0 (see the forward's tracer); compiled out unless
// FA_TRACE_BUILD is defined.
// FA_BTRACE_W: lane 0 of every gradient warp w = 4..11 into slice base + w - 4.
#ifdef FA_TRACE_BUILD
#define FA_BTRACE_DECL FA_TRACE_DECL
#define FA_BTRACE(who, ev, j) FA_TRACE(who, ev, j)
#define FA_BTRACE_WDECL                                                                              \
  unsigned trace_w = 0;                                                                              \
  unsigned long long* const trace_wp = blockIdx.x == 0 ? g_trace : nullptr
#define FA_BTRACE_W(base, ev, j)                                                                     \
  do {                                                                                               \
    if (trace_wp && (threadIdx.x & 31u) == 0 && trace_w < kTraceSlice)                               \
      trace_wp[((base) + threadIdx.x / 32 - 4) * kTraceSlice + trace_w++] =                          \
          (static_cast<unsigned long long>((ev) & 0xff) << 48) |                                    \
          (static_cast<unsigned long long>((j) & 0xffff) << 32) |                                   \
          (static_cast<unsigned long long>(clock64()) & 0xffffffffull);                             \
  } while (0)
#else
#define FA_BTRACE_DECL do { } while (0)
#define FA_BTRACE(who, ev, j) do { } while (0)
#define FA_BTRACE_WDECL do { } while (0)
#define FA_BTRACE_W(base, ev, j) do { } while (0)
#endif

// Exponentials of P taken on the FMA pipe: in blocks without masked keys,
// pairs i with i mod 8 >= 8 - FA_BWD_EMU of a thread's 32 take the degree-5
// polynomial (relative error 2.2e-7, like ex2.approx) instead of MUFU.  Off
// by default: measured on B200, 2, 3 and 4 of 8 were 0.6-2.8 % slower (the
// exponential unit does not bind the backward).
#ifndef FA_BWD_EMU
#define FA_BWD_EMU 0
#endif

// 2^x of pair i (i a compile-time constant after unrolling).
__device__ __forceinline__ float2 bwd_exp2_pair(float2 x, int i, bool emulate) {
  if (emulate && (i % 8) >= 8 - FA_BWD_EMU) return exp2_poly2<5>(x);
  return make_float2(ex2_approx(x.x), ex2_approx(x.y));
}

struct BwdParams {
  void* dk;                 // [B, N_k, H, D], 16-bit like the inputs
  void* dv;                 // [B, N_k, H, D]
  void* dq;                 // [B, N_q, H, D]
  const float* lse;         // [B, H, N_q] natural log (forward output)
  const float* delta;       // [B, H, N_q] rowsum(dO * O)
  int B, Nq, Nk, H;
  int Hkv, qpk;             // key/value heads; query head h reads K/V head h / qpk
  int causal;               // scheduling order only; the key bounds carry the mask
  int window_left;          // keys at most this many before the query; -1 = unlimited
  int window_right;         // keys at most this many after it; -1 = unlimited, 0 under
                            // causal (set by the host, below N_k + N_q < 2^31)
  // packed sequences (null cu_q: the padded batch [B, N_q / N_k, ...]):
  // sequence b owns rows cu_q[b] .. cu_q[b+1] of [total_q, H, D] (and of the
  // statistics [H, total_q]) and keys cu_k[b] .. cu_k[b+1] of [total_k, H_kv, D];
  // N_q / N_k are then the longest sequences
  const int* cu_q;
  const int* cu_k;
  int total_q, total_k;
  float scale;              // softmax scale
  float score_scale;        // scale * log2(e)
  int nkb;                  // key blocks per (batch, head)
  int nqb;                  // query blocks per (batch, head)
  unsigned long long wait_limit_ns;
  int* status;
  // dropout (DROP kernels): the forward's keep bits (keep_bits8 with these
  // values) and 1 / (1 - p)
  unsigned drop_threshold, seed_lo, seed_hi, drop_offset;
  PhiloxKeys drop_keys;     // the round keys of (seed_lo, seed_hi)
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
  // Q_i through three stages: S^T(n+1) wants Q_{n+1} early in visit n,
  // while Q_{n-1} is read until dK(n-1) at the end of visit n-1.  dO_i
  // through one: its first reader, dP^T(n+1), comes after its last, dV(n).
  static constexpr int OFF_Q = OFF_V + TILE;       // 3 stages of Q_i
  static constexpr int OFF_DO = OFF_Q + 3 * TILE;  // dO_i
  static constexpr int OFF_PT = OFF_DO + TILE;     // P^T, 128 keys x 128 queries
  static constexpr int SMEM = OFF_PT + 128 * 128 * 2;
  static constexpr int S_COL = 0, DP_COL = 128, DS_COL = 192;   // dS^T (16-bit) over dP^T's upper half
  static constexpr int DV_COL = 256, DK_COL = 256 + D;
  static_assert(SMEM <= 232448, "shared memory budget");
  static_assert(D == 64 || D == 128, "head dim");
};

struct BwdHeader {
  uint64_t kv_full;
  uint64_t q_full[3], q_empty[3];     // Q_i stages
  uint64_t do_full, do_empty;         // dO_i
  uint64_t s_full, dp_full;           // S^T, dP^T computed
  uint64_t s_free;                    // every gradient thread holds S^T in registers
  uint64_t p_ready;                   // P^T in shared memory
  uint64_t pt_free;                   // dV has read P^T
  uint64_t ds_ready;                  // dS^T in TMEM
  uint64_t dkv_full;                  // every MMA of the CTA done
  uint64_t stat_full[2], stat_empty[2];   // row statistics of a visit: loaded / read
  uint32_t tmem_base;
  int abort_flag;
  // -LSE * log2(e) (-inf: the row contributes nothing) and -D of the query
  // block, query q at stat_slot(q): the two half-warps, which read queries
  // e and 64 + e together, hit different banks and read four at a time
  alignas(16) float nlse2[2][128];
  alignas(16) float ndelta[2][128];
};

__device__ __forceinline__ int stat_slot(int q) { return ((q & 63) >> 2) * 8 + (q >> 6) * 4 + (q & 3); }
static_assert(sizeof(BwdHeader) <= 3072, "backward header");

constexpr int BWD_THREADS = 384;      // warpgroup 0: loads + MMA; warps 4-11: gradients

__device__ __forceinline__ void bwd_error(BwdHeader* sh, const BwdParams& p, int code) {
  atomicOr(p.status, code);
  atomicExch(&sh->abort_flag, 1);
}

__device__ __forceinline__ bool bwd_aborted(const int* flag) {
  return *reinterpret_cast<const volatile int*>(flag) != 0;
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

// One sequence of the batch: its sizes and where its rows start.  Packed
// sequences are clamped into the packed tensors (as in the forward), so bad
// offsets give wrong results but no access outside them.
struct BwdSeq {
  int nq, nk;            // queries and keys of the sequence
  int tq, tk, tb;        // TMA row of its first query / key, TMA batch coordinate
  long long qrow, krow;  // its first query / key row in [rows, heads, D]
  long long stat, stat_h;   // statistic of its first query for head 0, head stride
};

__device__ __forceinline__ BwdSeq bwd_seq(int b, const BwdParams& p) {
  BwdSeq s;
  if (p.cu_q) {
    const int q_start = min(max(__ldg(p.cu_q + b), 0), p.total_q);
    const int k_start = min(max(__ldg(p.cu_k + b), 0), p.total_k);
    s.nq = min(max(__ldg(p.cu_q + b + 1), q_start), p.total_q) - q_start;
    s.nk = min(max(__ldg(p.cu_k + b + 1), k_start), p.total_k) - k_start;
    s.tq = q_start;
    s.tk = k_start;
    s.tb = 0;
    s.qrow = q_start;
    s.krow = k_start;
    s.stat = q_start;
    s.stat_h = p.total_q;
  } else {
    s.nq = p.Nq;
    s.nk = p.Nk;
    s.tq = 0;
    s.tk = 0;
    s.tb = b;
    s.qrow = static_cast<long long>(b) * p.Nq;
    s.krow = static_cast<long long>(b) * p.Nk;
    s.stat = static_cast<long long>(b) * p.H * p.Nq;
    s.stat_h = p.Nq;
  }
  return s;
}

// Query blocks of a sequence of nq queries and nk keys that see key block
// jk: a right window (causal: 0) keeps queries at least window_right before
// the key (absolute indices), a left window keeps queries at most
// window_left after it.
__device__ __forceinline__ void bwd_query_range(int jk, const BwdParams& p, int nq, int nk, int& i_lo, int& i_hi) {
  const int nqb = (nq + 127) / 128;
  i_lo = p.window_right >= 0 ? max(0, jk * 128 - p.window_right) / 128 : 0;
  i_hi = nqb - 1;
  if (p.window_left >= 0) {
    const long long last = static_cast<long long>(jk) * 128 + 127 + p.window_left;
    i_hi = static_cast<int>(min(static_cast<long long>(i_hi), last / 128));
  }
  if (jk * 128 >= nk) i_hi = i_lo - 1;   // past the sequence's keys (packed batches)
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
  // so that head's Q and dO stay in L2 (longest first inside a head: for
  // causal attention key block 0 is seen by every query block).
  const int jk = static_cast<int>(blockIdx.x) % p.nkb;
  const int bhk = static_cast<int>(blockIdx.x) / p.nkb;   // (batch, K/V head)
  const int b = bhk / p.Hkv, hk = bhk - (bhk / p.Hkv) * p.Hkv;
  const BwdSeq sq = bwd_seq(b, p);
  int i_lo, i_hi;
  bwd_query_range(jk, p, sq.nq, sq.nk, i_lo, i_hi);
  // The n-th query block a CTA visits is i_lo + (n + rot) mod cnt: causal
  // CTAs already start at their own diagonal; the others start at a block
  // of their own, so CTAs running side by side read different Q blocks.
  const int cnt = i_hi - i_lo + 1;
  const int rot = (p.causal || cnt <= 0) ? 0 : jk % cnt;
  // every query head of the K/V head's group, cnt query blocks each: visit n
  // is query head hk * qpk + n / cnt, block i_lo + (n mod cnt + rot) mod cnt
  const int visits = cnt > 0 ? cnt * p.qpk : 0;
  const uint64_t lim = p.wait_limit_ns;

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&sh->kv_full), 1);
    for (int s = 0; s < 3; ++s) {
      mbar_init(smem_u32(&sh->q_full[s]), 1);
      mbar_init(smem_u32(&sh->q_empty[s]), 1);
    }
    mbar_init(smem_u32(&sh->do_full), 1);
    mbar_init(smem_u32(&sh->do_empty), 1);
    mbar_init(smem_u32(&sh->s_full), 1);
    mbar_init(smem_u32(&sh->s_free), 256);
    mbar_init(smem_u32(&sh->dp_full), 1);
    mbar_init(smem_u32(&sh->p_ready), 256);
    mbar_init(smem_u32(&sh->pt_free), 1);
    mbar_init(smem_u32(&sh->ds_ready), 256);
    mbar_init(smem_u32(&sh->dkv_full), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(smem_u32(&sh->stat_full[s]), 64);
      mbar_init(smem_u32(&sh->stat_empty[s]), 256);
    }
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
        tma_load_4d_hint(sbase + C::OFF_K + c * C::CHUNK, &tm_k, smem_u32(&sh->kv_full), c * 64, hk,
                         sq.tk + jk * 128, sq.tb, pol_kv);
        tma_load_4d_hint(sbase + C::OFF_V + c * C::CHUNK, &tm_v, smem_u32(&sh->kv_full), c * 64, hk,
                         sq.tk + jk * 128, sq.tb, pol_kv);
      }
      int nq = 0, nd = 0;   // Q and dO loads issued
      for (int n = 0; n < visits; ++n) {
        const int hq = hk * p.qpk + n / cnt;
        const int i = i_lo + (n % cnt + rot) % cnt;
        const int s = n % 3;
        if (!mbar_wait(smem_u32(&sh->q_empty[s]), ((n / 3) & 1) ^ 1, lim)) {
          bwd_error(sh, p, ST_TIMEOUT_LOAD);
          ok = false;
          break;
        }
        const uint32_t qbar = smem_u32(&sh->q_full[s]);
        mbar_arrive_expect_tx(qbar, C::TILE);
#pragma unroll
        for (int c = 0; c < C::NCHUNK; ++c)
          tma_load_4d_hint(sbase + C::OFF_Q + s * C::TILE + c * C::CHUNK, &tm_q, qbar, c * 64, hq, sq.tq + i * 128,
                           sq.tb, pol_q);
        ++nq;
        if (!mbar_wait(smem_u32(&sh->do_empty), (n & 1) ^ 1, lim)) {
          bwd_error(sh, p, ST_TIMEOUT_LOAD);
          ok = false;
          break;
        }
        const uint32_t dbar = smem_u32(&sh->do_full);
        mbar_arrive_expect_tx(dbar, C::TILE);
#pragma unroll
        for (int c = 0; c < C::NCHUNK; ++c)
          tma_load_4d_hint(sbase + C::OFF_DO + c * C::CHUNK, &tm_do, dbar, c * 64, hq, sq.tq + i * 128, sq.tb,
                           pol_q);
        ++nd;
      }
      if (!ok) {
        // drain: the copies already issued land before the CTA exits
        mbar_wait(smem_u32(&sh->kv_full), 0, lim);
        for (int m = max(0, nq - 3); m < nq; ++m) mbar_wait(smem_u32(&sh->q_full[m % 3]), (m / 3) & 1, lim);
        if (nd > 0) mbar_wait(smem_u32(&sh->do_full), (nd - 1) & 1, lim);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane_id() == 0 && i_lo <= i_hi) {
      FA_BTRACE_DECL;
      constexpr uint32_t FMT = DT == DT_BF16 ? 1u : 0u;
      constexpr uint32_t ID_ST = make_idesc(FMT, false, 128, 128);          // S^T, dP^T: both K-major
      constexpr uint32_t ID_KV = make_idesc(FMT, true, 128, D);             // dV, dK: B M/N-major
      constexpr uint32_t HI = sdesc_sw128_hi(1024);
      const uint32_t k_kmaj = sdesc_sw128_lo(sbase + C::OFF_K, 16);
      const uint32_t v_kmaj = sdesc_sw128_lo(sbase + C::OFF_V, 16);
      const uint32_t pt_kmaj = sdesc_sw128_lo(sbase + C::OFF_PT, 16);
      const uint32_t q_tile0 = sbase + C::OFF_Q, do_tile = sbase + C::OFF_DO;
      // S^T = K Q_n^T and dP^T = V dO_n^T for the n-th query block (keys on
      // the lanes); both K-major
      auto issue_kmaj = [&](uint32_t col, uint32_t a_kmaj, uint32_t b_tile) {
        const uint32_t b_kmaj = sdesc_sw128_lo(b_tile, 16);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int byte = kk * 32;
          const uint32_t off = static_cast<uint32_t>(((byte / 128) * C::CHUNK + (byte % 128)) >> 4);
          mma_f16_ss_lo(tbase + col, a_kmaj + off, b_kmaj + off, HI, ID_ST, kk > 0);
        }
      };
      // Per query block n, in pipe order: S^T(n+1) (as soon as the gradient
      // warps hold S^T(n) in registers), dV(n) on P^T(n), dK(n) on dS^T(n),
      // then dP^T(n+1) over dP^T(n) and dS^T(n).  The gradient warps form
      // P(n+1) while dV(n), dK(n) and dP^T(n+1) run.
      bool ok = mbar_wait(smem_u32(&sh->kv_full), 0, lim) && mbar_wait(smem_u32(&sh->q_full[0]), 0, lim) &&
                mbar_wait(smem_u32(&sh->do_full), 0, lim);
      if (ok && visits > 0) {
        tc_fence_after();
        issue_kmaj(C::S_COL, k_kmaj, q_tile0);
        mma_commit(smem_u32(&sh->s_full));
        issue_kmaj(C::DP_COL, v_kmaj, do_tile);
        mma_commit(smem_u32(&sh->dp_full));
      }
      for (int n = 0; n < visits && ok; ++n) {
        const uint32_t q_tile = q_tile0 + (n % 3) * C::TILE;
        if (n + 1 < visits) {
          FA_BTRACE(2, 0, n);
          if (!mbar_wait(smem_u32(&sh->s_free), n & 1, lim) ||
              !mbar_wait(smem_u32(&sh->q_full[(n + 1) % 3]), ((n + 1) / 3) & 1, lim)) {
            ok = false;
            break;
          }
          FA_BTRACE(2, 1, n);
          tc_fence_after();
          issue_kmaj(C::S_COL, k_kmaj, q_tile0 + ((n + 1) % 3) * C::TILE);
          mma_commit(smem_u32(&sh->s_full));
        }
        if (!mbar_wait(smem_u32(&sh->p_ready), n & 1, lim)) { ok = false; break; }
        FA_BTRACE(2, 2, n);
        tc_fence_after();
        const uint32_t q_mn = sdesc_sw128_lo(q_tile, C::CHUNK), do_mn = sdesc_sw128_lo(do_tile, C::CHUNK);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          // dV += P^T dO_n: A = P^T in shared memory, K-major (16 queries = 32 bytes of a row)
          const int byte = kk * 32;
          const uint32_t a_off = static_cast<uint32_t>(((byte / 128) * C::CHUNK + (byte % 128)) >> 4);
          const uint32_t b_off = static_cast<uint32_t>((kk * 16 * 128) >> 4);
          mma_f16_ss_lo(tbase + C::DV_COL, pt_kmaj + a_off, do_mn + b_off, HI, ID_KV, n > 0 || kk > 0);
        }
        mma_commit(smem_u32(&sh->pt_free));
        mma_commit(smem_u32(&sh->do_empty));   // dV(n) is dO_n's last reader
        if (!mbar_wait(smem_u32(&sh->ds_ready), n & 1, lim)) { ok = false; break; }
        FA_BTRACE(2, 3, n);
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          // dK += dS^T Q_n: A = dS^T (16-bit) in TMEM, 16 queries = 8 columns per step
          const uint32_t off = static_cast<uint32_t>((kk * 16 * 128) >> 4);
          mma_f16_ts_lo(tbase + C::DK_COL, tbase + C::DS_COL + kk * 8, q_mn + off, HI, ID_KV, n > 0 || kk > 0);
        }
        mma_commit(smem_u32(&sh->q_empty[n % 3]));   // dK(n) is Q_n's last reader
        if (n + 1 < visits) {
          if (!mbar_wait(smem_u32(&sh->do_full), (n + 1) & 1, lim)) { ok = false; break; }
          tc_fence_after();
          issue_kmaj(C::DP_COL, v_kmaj, do_tile);
          mma_commit(smem_u32(&sh->dp_full));
        }
        FA_BTRACE(2, 4, n);
      }
      if (!ok) bwd_error(sh, p, ST_TIMEOUT_MMA);
      mma_commit(smem_u32(&sh->dkv_full));   // also: every MMA done before TMEM is released
      if (!ok) mbar_wait(smem_u32(&sh->dkv_full), 0, lim);
    }
  } else if (warp < 4) {
    // ---------------------------------------------------- row statistics
    // Warps 2-3 load, per visit, -LSE log2(e) and -D of the query block's
    // 128 rows (two per thread) into stat buffer n mod 2, once the gradient
    // warps have released it (rows past N_q: -inf and 0, so they contribute
    // nothing)
    const int u = static_cast<int>(threadIdx.x) - 64;   // 0..63
    int qn = 0, ib = 0;   // visit n = qn * cnt + ib: query head hk * qpk + qn, block (ib + rot) mod cnt
    for (int n = 0; n < visits; ++n) {
      const int s = n & 1;
      if (!mbar_wait(smem_u32(&sh->stat_empty[s]), ((n >> 1) & 1) ^ 1, lim)) {
        if (u == 0) bwd_error(sh, p, ST_TIMEOUT_LOAD);
        break;
      }
      const int hq = hk * p.qpk + qn;
      const int i = i_lo + (ib + rot < cnt ? ib + rot : ib + rot - cnt);
      const long long base = sq.stat + hq * sq.stat_h;
#pragma unroll
      for (int x = 0; x < 2; ++x) {
        const int ql = 2 * u + x, q = i * 128 + ql;
        float nl = -INFINITY, nd = 0.f;
        if (q < sq.nq) {
          const float l = p.lse[base + q];
          if (l != -INFINITY) nl = l * -1.4426950408889634f;
          nd = -p.delta[base + q];
        }
        sh->nlse2[s][stat_slot(ql)] = nl;
        sh->ndelta[s][stat_slot(ql)] = nd;
      }
      mbar_arrive(smem_u32(&sh->stat_full[s]));   // release: the stores above are seen after the wait
      if (++ib == cnt) { ib = 0; ++qn; }
    }
  } else {
    // ---------------------------------------------------------- gradients
    const int quad = warp & 3;
    const int sub = (warp - 4) >> 2;
    const int lane = static_cast<int>(lane_id());
    const int half = lane >> 4;
    const int r = quad * 32 + sub * 16 + (lane & 15);           // TMEM lane: key
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32 + sub * 16) << 16;
    const int key = jk * 128 + r;
    const float c2 = p.score_scale;
    uint8_t* pt_row = smem + C::OFF_PT + half * C::CHUNK + r * 128;
    // Each warp takes its own exit decision: a wait that runs out records
    // the error and raises the CTA's abort flag, which every warp checks
    // once per visit (all waits are bounded, so no warp is left behind for
    // long); the vote after the loop then agrees on the outcome.
    bool ok = true;
    FA_BTRACE_DECL;
    FA_BTRACE_WDECL;
    int qn = 0, ib = 0;   // visit n = qn * cnt + ib
    for (int n = 0; n < visits; ++n) {
      FA_BTRACE(0, 0, n);
      FA_BTRACE_W(4, 0, n);
      if (__any_sync(0xffffffffu, bwd_aborted(&sh->abort_flag))) { ok = false; break; }
      const int hq = hk * p.qpk + qn;
      const int i = i_lo + (ib + rot < cnt ? ib + rot : ib + rot - cnt);
      if (++ib == cnt) { ib = 0; ++qn; }
      const int buf = n & 1;
      const int q0 = i * 128;
      const bool need_mask = (jk * 128 + 128 > sq.nk) || (p.window_right >= 0 && jk * 128 + 127 > q0 + p.window_right) ||
                             (p.window_left >= 0 && jk * 128 < q0 + 127 - p.window_left);
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
          const uint32_t mine8 = keep_bits8(grp, qq, bh, p.drop_offset, p.drop_keys, p.drop_threshold);
          uint32_t got8 = 0;
#pragma unroll
          for (int x = 0; x < 8; ++x) {
            const uint32_t v8 = __shfl_sync(0xffffffffu, mine8, (lane & ~7) + x);
            got8 |= ((v8 >> lane8) & 1u) << x;
          }
          keep[m / 4] |= got8 << (8 * (m % 4));
        }
      }
      FA_BTRACE_W(4, 1, n);
      if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&sh->s_full), n & 1, lim) &&
                                       mbar_wait(smem_u32(&sh->stat_full[buf]), (n >> 1) & 1, lim))) {
        if (lane == 0) bwd_error(sh, p, ST_TIMEOUT_SOFTMAX);
        ok = false;
        break;
      }
      FA_BTRACE_W(4, 2, n);
      FA_BTRACE(0, 1, n);
      FA_BTRACE_W(4, 3, n);
      tc_fence_after();
      // the thread's half row of S^T (queries half * 64 + [0, 64)); the MMA
      // may overwrite S^T with the next block's once every thread has it
      float pv[64];
      tmem_ld_16x32bx2_x32<64>(tbase + lane_off + C::S_COL, reinterpret_cast<uint32_t*>(pv));
      tmem_ld_16x32bx2_x32<64>(tbase + lane_off + C::S_COL + 32, reinterpret_cast<uint32_t*>(pv + 32));
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(smem_u32(&sh->s_free));
      if (need_mask) {
        // keys a query may not see: a score of -inf gives P = 0
#pragma unroll
        for (int e = 0; e < 64; ++e) {
          const int q = q0 + half * 64 + e;
          const bool vis = key < sq.nk && (p.window_right < 0 || key <= q + p.window_right) &&
                           (p.window_left < 0 || key >= q - p.window_left);
          pv[e] = vis ? pv[e] : -INFINITY;
        }
      }
      // P = 2^(S c2 - LSE log2 e), the statistic held negated; queries
      // e..e+3 at [2 (e / 4)].  Two copies of the loop, so that no branch
      // sits between its exponentials
      const float4* nl4 = reinterpret_cast<const float4*>(sh->nlse2[buf]) + half;
      const float2 c2v = make_float2(c2, c2);
      auto p_block = [&](bool emulate) {
#pragma unroll
        for (int e4 = 0; e4 < 16; ++e4) {
          const float4 l4 = nl4[2 * e4];
          const float2 x0 = __ffma2_rn(make_float2(pv[4 * e4], pv[4 * e4 + 1]), c2v, make_float2(l4.x, l4.y));
          const float2 x1 = __ffma2_rn(make_float2(pv[4 * e4 + 2], pv[4 * e4 + 3]), c2v, make_float2(l4.z, l4.w));
          const float2 y0 = bwd_exp2_pair(x0, 2 * e4, emulate), y1 = bwd_exp2_pair(x1, 2 * e4 + 1, emulate);
          pv[4 * e4] = y0.x, pv[4 * e4 + 1] = y0.y, pv[4 * e4 + 2] = y1.x, pv[4 * e4 + 3] = y1.y;
        }
      };
      if (need_mask) p_block(false);
      else p_block(true);
      FA_BTRACE(0, 2, n);
      // P^T(n - 1) in shared memory has been read by dV(n - 1)
      if (n > 0 && !__all_sync(0xffffffffu, mbar_wait(smem_u32(&sh->pt_free), (n - 1) & 1, lim))) {
        if (lane == 0) bwd_error(sh, p, ST_TIMEOUT_SOFTMAX);
        ok = false;
        break;
      }
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        // P^T for queries half * 64 + [16c, 16c + 16) (dV takes the kept
        // probabilities, scaled by 1 / (1 - p)): row r, two 16-byte units of
        // the 128-byte row, XOR-swizzled by (r mod 8) like a TMA 128B tile
        uint32_t pw[8];
#pragma unroll
        for (int e = 0; e < 16; e += 2) {
          float p0 = pv[c * 16 + e], p1 = pv[c * 16 + e + 1];
          if constexpr (DROP) {
            const uint32_t kb = keep[(c * 16 + e) / 32] >> ((c * 16 + e) % 32);
            p0 = (kb & 1u) ? p0 * p.drop_scale : 0.f;
            p1 = (kb & 2u) ? p1 * p.drop_scale : 0.f;
          }
          pw[e / 2] = pack2<DT>(p0, p1);
        }
        const int u0 = (2 * c) ^ (r & 7), u1 = (2 * c + 1) ^ (r & 7);
        *reinterpret_cast<uint4*>(pt_row + u0 * 16) = make_uint4(pw[0], pw[1], pw[2], pw[3]);
        *reinterpret_cast<uint4*>(pt_row + u1 * 16) = make_uint4(pw[4], pw[5], pw[6], pw[7]);
      }
      fence_proxy_async_smem();   // P^T stores visible to the MMA's reads
      mbar_arrive(smem_u32(&sh->p_ready));
      // dP^T(n): the warp reads all of it before any dS^T store lands over
      // its upper half
      if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&sh->dp_full), n & 1, lim))) {
        if (lane == 0) bwd_error(sh, p, ST_TIMEOUT_SOFTMAX);
        ok = false;
        break;
      }
      FA_BTRACE(0, 3, n);
      tc_fence_after();
      float gv[64];
      tmem_ld_16x32bx2_x32<64>(tbase + lane_off + C::DP_COL, reinterpret_cast<uint32_t*>(gv));
      tmem_ld_16x32bx2_x32<64>(tbase + lane_off + C::DP_COL + 32, reinterpret_cast<uint32_t*>(gv + 32));
      tmem_wait_ld();
      const float4* nd4 = reinterpret_cast<const float4*>(sh->ndelta[buf]) + half;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t dw[16];
#pragma unroll
        for (int e4 = 0; e4 < 8; ++e4) {
          const float4 v4 = nd4[2 * (8 * c + e4)];
#pragma unroll
          for (int x = 0; x < 4; x += 2) {
            const int e = 32 * c + 4 * e4 + x;
            float2 g = make_float2(gv[e], gv[e + 1]);
            if constexpr (DROP) {
              // dP of the dropped forward: Z / (1 - p) times dO V^T
              const uint32_t kb = keep[c] >> ((4 * e4 + x) % 32);
              g.x = (kb & 1u) ? g.x * p.drop_scale : 0.f;
              g.y = (kb & 2u) ? g.y * p.drop_scale : 0.f;
            }
            const float2 nd = x == 0 ? make_float2(v4.x, v4.y) : make_float2(v4.z, v4.w);
            const float2 d = __fmul2_rn(make_float2(pv[e], pv[e + 1]), __fadd2_rn(g, nd));
            dw[(4 * e4 + x) / 2] = pack2<DT>(d.x, d.y);
          }
        }
        // dS^T (16-bit) for the thread's queries 32c .. 32c + 31: columns
        // DS_COL + 16c (+ 32 for the upper half-warp)
        tmem_st_16x32bx2_x16<32>(tbase + lane_off + C::DS_COL + c * 16, dw);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(smem_u32(&sh->ds_ready));
      mbar_arrive(smem_u32(&sh->stat_empty[buf]));   // this visit's statistics read
      FA_BTRACE(0, 4, n);
      FA_BTRACE_W(4, 4, n);
    }
    if (!grad_bar_and(ok)) {
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
      const long long row = (sq.krow + key) * p.Hkv + hk;
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
        if (key < sq.nk) {
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
// query blocks with the most keys first.  Warp 0 loads Q_i and dO_i once,
// then K_j and V_j through their stages (below); warp 1 issues
// S = Q_i K_j^T and dP = dO_i V_j^T (queries on the lanes) and, on dS(j),
// dQ += dS K_j with A = dS from TMEM; warps 4-11 form dS = P * (dP - D) with
// P = exp(S - LSE).  S is double-buffered in TMEM, so the gradient warps
// form P(j+1) while the tensor pipe runs dP(j+1), dQ(j) and S(j+2): per key
// block the MMA thread issues, after dS(j), dP(j+1) (over dP(j), read by
// then), dQ(j), and S(j+2) into the buffer of S(j) (whose dS(j) dQ(j) has
// read, in pipe order).
// TMEM: S(even) [0,128), dP [128,256), dQ [256,256+D), S(odd) [384,512);
// dS (16-bit) over the upper half of its S buffer.
// K and V stages: K_j is read until dQ(j), V_j only by dP(j), and the two
// share five tile slots; four K stages and one V stage measured 0.3 % ahead
// of three and two (S(j+2) no longer waits for K_{j+2} to land).
#ifndef FA_DQ_KSTAGES
#define FA_DQ_KSTAGES 4
#endif

struct DqHeader {
  uint64_t q_full;
  uint64_t k_full[4], k_empty[4];
  uint64_t v_full[2], v_empty[2];
  uint64_t s_full[2];        // S(j) in buffer j mod 2 computed
  uint64_t dp_full;          // dP(j) computed
  uint64_t ds_ready;         // dS(j) in TMEM
  uint64_t dq_done;          // every MMA done
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(DqHeader) <= 1024, "dQ header");

__device__ __forceinline__ void dq_error(DqHeader* sh, const BwdParams& p, int code) {
  atomicOr(p.status, code);
  atomicExch(&sh->abort_flag, 1);
}

template <int D>
struct DqCfg {
  static constexpr int TILE = BwdCfg<D>::TILE;
  static constexpr int OFF_Q = 1024, OFF_DO = OFF_Q + TILE;
  static constexpr int KS = FA_DQ_KSTAGES, VS = 5 - FA_DQ_KSTAGES;   // K and V stages
  static constexpr int OFF_K = OFF_DO + TILE;
  static constexpr int OFF_V = OFF_K + KS * TILE;
  static constexpr int SMEM_USED = OFF_V + VS * TILE;
  static constexpr uint32_t S_COL0 = 0, S_COL1 = 384, DP_COL = 128, DQ_COL = 256;
  static_assert(SMEM_USED <= 232448, "shared memory budget");
};

template <int D, int DT, bool DROP>
__global__ void __launch_bounds__(BWD_THREADS, 1)
    fa_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                     const BwdParams p) {
  using C = BwdCfg<D>;
  using Q = DqCfg<D>;
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
  const BwdSeq sq = bwd_seq(b, p);
  const int q0 = iq * 128;
  // key blocks the rows of this query block see (as in the forward)
  const int qe = min(q0 + 127, sq.nq - 1);
  const int j_lo = p.window_left >= 0 ? max(0, q0 - p.window_left) / 128 : 0;
  const int j_hi = p.window_right >= 0 ? min(qe + p.window_right, sq.nk - 1) / 128 : (sq.nk - 1) / 128;
  const int cnt = (q0 < sq.nq && sq.nk > 0) ? max(0, j_hi - j_lo + 1) : 0;
  const uint64_t lim = p.wait_limit_ns;

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&sh->q_full), 1);
    for (int s = 0; s < Q::KS; ++s) {
      mbar_init(smem_u32(&sh->k_full[s]), 1);
      mbar_init(smem_u32(&sh->k_empty[s]), 1);
    }
    for (int s = 0; s < Q::VS; ++s) {
      mbar_init(smem_u32(&sh->v_full[s]), 1);
      mbar_init(smem_u32(&sh->v_empty[s]), 1);
    }
    for (int s = 0; s < 2; ++s) mbar_init(smem_u32(&sh->s_full[s]), 1);
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
        tma_load_4d_hint(sbase + Q::OFF_Q + c * C::CHUNK, &tm_q, smem_u32(&sh->q_full), c * 64, h, sq.tq + q0, sq.tb,
                         pol_q);
        tma_load_4d_hint(sbase + Q::OFF_DO + c * C::CHUNK, &tm_do, smem_u32(&sh->q_full), c * 64, h, sq.tq + q0,
                         sq.tb, pol_q);
      }
      int nk = 0, nv = 0;   // K and V loads issued
      for (int n = 0; n < cnt && ok; ++n) {
        const int j = j_lo + n;
        const int sk = n % Q::KS, sv = n % Q::VS;
        if (!mbar_wait(smem_u32(&sh->k_empty[sk]), ((n / Q::KS) & 1) ^ 1, lim)) { ok = false; break; }
        mbar_arrive_expect_tx(smem_u32(&sh->k_full[sk]), C::TILE);
#pragma unroll
        for (int c = 0; c < C::NCHUNK; ++c)
          tma_load_4d_hint(sbase + Q::OFF_K + sk * C::TILE + c * C::CHUNK, &tm_k, smem_u32(&sh->k_full[sk]), c * 64,
                           hk, sq.tk + j * 128, sq.tb, pol_kv);
        ++nk;
        if (!mbar_wait(smem_u32(&sh->v_empty[sv]), ((n / Q::VS) & 1) ^ 1, lim)) { ok = false; break; }
        mbar_arrive_expect_tx(smem_u32(&sh->v_full[sv]), C::TILE);
#pragma unroll
        for (int c = 0; c < C::NCHUNK; ++c)
          tma_load_4d_hint(sbase + Q::OFF_V + sv * C::TILE + c * C::CHUNK, &tm_v, smem_u32(&sh->v_full[sv]), c * 64,
                           hk, sq.tk + j * 128, sq.tb, pol_kv);
        ++nv;
      }
      if (!ok) {
        // drain: the copies already issued land before the CTA exits
        dq_error(sh, p, ST_TIMEOUT_LOAD);
        mbar_wait(smem_u32(&sh->q_full), 0, lim);
        for (int m = max(0, nk - Q::KS); m < nk; ++m) mbar_wait(smem_u32(&sh->k_full[m % Q::KS]), (m / Q::KS) & 1, lim);
        for (int m = max(0, nv - Q::VS); m < nv; ++m) mbar_wait(smem_u32(&sh->v_full[m % Q::VS]), (m / Q::VS) & 1, lim);
      }
    }
  } else if (warp == 1) {
    if (lane_id() == 0 && cnt > 0) {
      FA_BTRACE_DECL;
      constexpr uint32_t FMT = DT == DT_BF16 ? 1u : 0u;
      constexpr uint32_t ID_S = make_idesc(FMT, false, 128, 128);   // S, dP: both K-major
      constexpr uint32_t ID_Q = make_idesc(FMT, true, 128, D);      // dQ: A in TMEM, B head-dim-major
      constexpr uint32_t HI = sdesc_sw128_hi(1024);
      const uint32_t q_kmaj = sdesc_sw128_lo(sbase + Q::OFF_Q, 16);
      const uint32_t do_kmaj = sdesc_sw128_lo(sbase + Q::OFF_DO, 16);
      // S(n) = Q K_n^T into buffer n mod 2, on K_n landed
      auto issue_s = [&](int n) -> bool {
        if (!mbar_wait(smem_u32(&sh->k_full[n % Q::KS]), (n / Q::KS) & 1, lim)) return false;
        FA_BTRACE(12, 6, n);
        tc_fence_after();
        const uint32_t k_kmaj = sdesc_sw128_lo(sbase + Q::OFF_K + (n % Q::KS) * C::TILE, 16);
        const uint32_t col = (n & 1) ? Q::S_COL1 : Q::S_COL0;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int byte = kk * 32;
          const uint32_t off = static_cast<uint32_t>(((byte / 128) * C::CHUNK + (byte % 128)) >> 4);
          mma_f16_ss_lo(tbase + col, q_kmaj + off, k_kmaj + off, HI, ID_S, kk > 0);
        }
        FA_BTRACE(12, 7, n);
        mma_commit(smem_u32(&sh->s_full[n & 1]));
        return true;
      };
      // dP(n) = dO V_n^T, on V_n landed; V_n's stage is free after it
      auto issue_dp = [&](int n) -> bool {
        if (!mbar_wait(smem_u32(&sh->v_full[n % Q::VS]), (n / Q::VS) & 1, lim)) return false;
        FA_BTRACE(12, 4, n);
        tc_fence_after();
        const uint32_t v_kmaj = sdesc_sw128_lo(sbase + Q::OFF_V + (n % Q::VS) * C::TILE, 16);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int byte = kk * 32;
          const uint32_t off = static_cast<uint32_t>(((byte / 128) * C::CHUNK + (byte % 128)) >> 4);
          mma_f16_ss_lo(tbase + Q::DP_COL, do_kmaj + off, v_kmaj + off, HI, ID_S, kk > 0);
        }
        FA_BTRACE(12, 5, n);
        mma_commit(smem_u32(&sh->dp_full));
        mma_commit(smem_u32(&sh->v_empty[n % Q::VS]));
        return true;
      };
      bool ok = mbar_wait(smem_u32(&sh->q_full), 0, lim) && issue_s(0) && issue_dp(0) && (cnt < 2 || issue_s(1));
      for (int n = 0; n < cnt && ok; ++n) {
        FA_BTRACE(12, 0, n);
        if (!mbar_wait(smem_u32(&sh->ds_ready), n & 1, lim)) { ok = false; break; }
        FA_BTRACE(12, 1, n);
        tc_fence_after();
        // dP(n+1) over dP(n): the gradient warps read dP(n) before dS(n)
        if (n + 1 < cnt && !issue_dp(n + 1)) { ok = false; break; }
        // dQ += dS K_n: A = dS (16-bit, upper half of S(n)'s buffer), 16 keys = 8 columns per step
        const uint32_t k_mn = sdesc_sw128_lo(sbase + Q::OFF_K + (n % Q::KS) * C::TILE, C::CHUNK);
        const uint32_t ds_col = ((n & 1) ? Q::S_COL1 : Q::S_COL0) + 64;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = static_cast<uint32_t>((kk * 16 * 128) >> 4);
          mma_f16_ts_lo(tbase + Q::DQ_COL, tbase + ds_col + kk * 8, k_mn + off, HI, ID_Q, n > 0 || kk > 0);
        }
        mma_commit(smem_u32(&sh->k_empty[n % Q::KS]));   // last reader of K_n
        FA_BTRACE(12, 2, n);
        // S(n+2) over S(n) and dS(n), after dQ(n) (same pipe, in order)
        if (n + 2 < cnt && !issue_s(n + 2)) { ok = false; break; }
        FA_BTRACE(12, 3, n);
      }
      if (!ok) dq_error(sh, p, ST_TIMEOUT_MMA);
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
    const long long bhq = sq.stat + h * sq.stat_h;
    // this row's statistics: -LSE * log2(e) (-inf: the row contributes nothing) and D
    float nlse2 = -INFINITY, dlt = 0.f;
    if (q < sq.nq) {
      const float l = p.lse[bhq + q];
      if (l != -INFINITY) nlse2 = l * -1.4426950408889634f;
      dlt = p.delta[bhq + q];
    }
    const float c2 = p.score_scale;
    // Each warp takes its own exit decision (see the dK/dV kernel); the
    // vote after the loop agrees on the outcome
    bool ok = true;
    FA_BTRACE_DECL;
    FA_BTRACE_WDECL;
    for (int n = 0; n < cnt; ++n) {
      if (threadIdx.x == 128) FA_BTRACE(3, 0, n);
      FA_BTRACE_W(16, 0, n);
      if (__any_sync(0xffffffffu, bwd_aborted(&sh->abort_flag))) { ok = false; break; }
      const int k0 = (j_lo + n) * 128;
      const uint32_t s_col = (n & 1) ? Q::S_COL1 : Q::S_COL0;
      const bool need_mask = (k0 + 128 > sq.nk) || (p.window_right >= 0 && k0 + 127 > q0 + p.window_right) ||
                             (p.window_left >= 0 && k0 < q0 + 127 - p.window_left);
      // dropout keep bits of this row's keys k0 + 64 * half + [0, 64)
      uint32_t keep[2] = {0u, 0u};
      if constexpr (DROP) {
        const uint32_t g0 = static_cast<uint32_t>(k0 + half * 64) / 8u;
        const uint32_t bhq = static_cast<uint32_t>(b * p.H + h);
#pragma unroll
        for (int g = 0; g < 8; ++g)
          keep[g / 4] |= keep_bits8(g0 + g, static_cast<uint32_t>(q), bhq, p.drop_offset, p.drop_keys,
                                    p.drop_threshold)
                         << (8 * (g % 4));
      }
      FA_BTRACE_W(16, 1, n);
      if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&sh->s_full[n & 1]), (n >> 1) & 1, lim))) {
        if (lane == 0) dq_error(sh, p, ST_TIMEOUT_SOFTMAX);
        ok = false;
        break;
      }
      FA_BTRACE_W(16, 2, n);
      if (threadIdx.x == 128) FA_BTRACE(3, 1, n);
      FA_BTRACE_W(16, 3, n);
      tc_fence_after();
      // the whole half row of S (keys half * 64 + [0, 64)) before any dS store
      float pv[64];
      tmem_ld_16x32bx2_x32<64>(tbase + lane_off + s_col, reinterpret_cast<uint32_t*>(pv));
      tmem_ld_16x32bx2_x32<64>(tbase + lane_off + s_col + 32, reinterpret_cast<uint32_t*>(pv + 32));
      tmem_wait_ld();
      if (need_mask) {
        // keys the row may not see: a score of -inf gives P = 0
#pragma unroll
        for (int e = 0; e < 64; ++e) {
          const int key = k0 + half * 64 + e;
          const bool vis = key < sq.nk && (p.window_right < 0 || key <= q + p.window_right) &&
                           (p.window_left < 0 || key >= q - p.window_left);
          pv[e] = vis ? pv[e] : -INFINITY;
        }
      }
      // P = 2^(S c2 - LSE log2 e); two copies of the loop, so that no
      // branch sits between its exponentials
      const float2 c2v = make_float2(c2, c2), nl2 = make_float2(nlse2, nlse2);
      auto p_block = [&](bool emulate) {
#pragma unroll
        for (int e = 0; e < 64; e += 2) {
          const float2 y = bwd_exp2_pair(__ffma2_rn(make_float2(pv[e], pv[e + 1]), c2v, nl2), e / 2, emulate);
          pv[e] = y.x, pv[e + 1] = y.y;
        }
      };
      if (need_mask) p_block(false);
      else p_block(true);
      if (threadIdx.x == 128) FA_BTRACE(3, 2, n);
      // dP(n)
      if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&sh->dp_full), n & 1, lim))) {
        if (lane == 0) dq_error(sh, p, ST_TIMEOUT_SOFTMAX);
        ok = false;
        break;
      }
      tc_fence_after();
      float gv[64];
      tmem_ld_16x32bx2_x32<64>(tbase + lane_off + Q::DP_COL, reinterpret_cast<uint32_t*>(gv));
      tmem_ld_16x32bx2_x32<64>(tbase + lane_off + Q::DP_COL + 32, reinterpret_cast<uint32_t*>(gv + 32));
      tmem_wait_ld();
      const float2 nd2 = make_float2(-dlt, -dlt);
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t dw[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          float2 g = make_float2(gv[32 * c + e], gv[32 * c + e + 1]);
          if constexpr (DROP) {
            // dP of the dropped forward: Z / (1 - p) times dO V^T
            const uint32_t kb = keep[c] >> e;
            g.x = (kb & 1u) ? g.x * p.drop_scale : 0.f;
            g.y = (kb & 2u) ? g.y * p.drop_scale : 0.f;
          }
          const float2 d = __fmul2_rn(make_float2(pv[32 * c + e], pv[32 * c + e + 1]), __fadd2_rn(g, nd2));
          dw[e / 2] = pack2<DT>(d.x, d.y);
        }
        // dS for the thread's keys 32c .. 32c + 31 over S(n)'s upper half
        tmem_st_16x32bx2_x16<32>(tbase + lane_off + s_col + 64 + c * 16, dw);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(smem_u32(&sh->ds_ready));
      if (threadIdx.x == 128) FA_BTRACE(3, 3, n);
      FA_BTRACE_W(16, 4, n);
    }
    if (!grad_bar_and(ok)) {
      ok = false;
      if (threadIdx.x == 128) atomicOr(p.status, ST_TIMEOUT_SOFTMAX);
    }
    // dQ = scale * (sum over key blocks of dS K), 16-bit
    bool have = ok && cnt > 0;
    if (have) {
      have = __all_sync(0xffffffffu, mbar_wait(smem_u32(&sh->dq_done), 0, lim));
      if (!have && lane == 0) atomicOr(p.status, ST_TIMEOUT_SOFTMAX);
      tc_fence_after();
    }
    // (the TMEM loads are warp-collective: every lane takes them, whatever
    // its row; only rows inside N_q are stored)
    if (have || (ok && cnt == 0)) {
      uint8_t* dq_row = reinterpret_cast<uint8_t*>(p.dq) +
                        (((sq.qrow + q) * p.H + h) * D + half * (D / 2)) * 2;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t v[16];
        if (cnt > 0) {
          tmem_ld_16x32bx2_x16<D / 2>(tbase + lane_off + Q::DQ_COL + c * 16, v);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int e = 0; e < 16; ++e) v[e] = 0u;
        }
        if (q < sq.nq) store_out_row16<DT>(dq_row + c * 32, reinterpret_cast<const float*>(v), p.scale);
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

// D_i = sum_d dO_id O_id (fp32) for every (b, h, i).  Each thread reads 16
// bytes of O and of dO (8 elements); the D / 8 threads of a row add theirs
// with shuffles.  Whole warps step through the grid-stride loop together.
template <int D>
__global__ void fa_bwd_prologue_kernel(const void* __restrict__ out, const void* __restrict__ dout, int dt,
                                       float* __restrict__ delta, int B, int Nq, int H) {
  constexpr int TPR = D / 8;   // threads per row
  const long long total = static_cast<long long>(B) * Nq * H * TPR;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  const int lane = static_cast<int>(threadIdx.x & 31u);
  const uint4* o4 = reinterpret_cast<const uint4*>(out);
  const uint4* g4 = reinterpret_cast<const uint4*>(dout);
  for (long long g = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; g - lane < total; g += stride) {
    float acc = 0.f;
    if (g < total) {
      const uint4 ov = __ldg(o4 + g), gv = __ldg(g4 + g);
      const uint32_t ow[4] = {ov.x, ov.y, ov.z, ov.w}, gw[4] = {gv.x, gv.y, gv.z, gv.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float2 of, gf;
        if (dt == DT_BF16) {
          of = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ow[e]));
          gf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&gw[e]));
        } else {
          of = __half22float2(*reinterpret_cast<const __half2*>(&ow[e]));
          gf = __half22float2(*reinterpret_cast<const __half2*>(&gw[e]));
        }
        acc = fmaf(of.x, gf.x, acc);
        acc = fmaf(of.y, gf.y, acc);
      }
    }
#pragma unroll
    for (int m = TPR / 2; m > 0; m >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, m);
    if (g < total && (lane % TPR) == 0) {
      // row g / TPR enumerates (b, n, h); D_i is stored [B, H, N_q] like the LSE
      const long long i = g / TPR;
      const long long h = i % H, bn = i / H, nq = bn % Nq, bb = bn / Nq;
      delta[(bb * H + h) * Nq + nq] = acc;
    }
  }
}

}  // namespace fa
