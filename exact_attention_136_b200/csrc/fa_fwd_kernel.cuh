// Exact attention forward for sm_100a: O = softmax(scale * Q K^T + mask) V
// and LSE = log(sum_j exp(scale * q.k_j)), with the N x N scores kept on chip.
//
// What is computed follows the Flash Attention skill pages (Flash Attention |
// Hermes Skill, Workflow 1 Step 2 "standard attention"; Workflow 2 Steps 2-3
// for causal=True and window_size=(left, right)); how it is tiled follows the
// explainer "FlashAttention" (aiunderstanding.org, "Technical insight"): small
// blocks of queries, keys and values in on-chip memory, an online softmax
// that rescales running sums as new key blocks arrive, one fused kernel.
//
// B200 design (one CTA per SM, persistent over work units):
//   work unit  = (batch b, head h, 256 query rows) = two 128-row Q tiles.
//   warp 0     : TMA producer.  Q0/Q1 once per unit, then K_j, V_j tiles of
//                128 keys through a ring of shared-memory slots (mbarrier
//                full/empty pairs).
//   warp 1     : owns TMEM (512 columns) and issues every tcgen05.mma from
//                one thread:  S_t = Q_t K_j^T  (SS, fp32 accumulate in TMEM)
//                and O_t += P_t V_j (TS: P read from TMEM, V from smem).
//                Per key block j the issue order is
//                  PV_0(j-1), S_0(j), PV_1(j-1), S_1(j)
//                so the tensor pipe works on one tile while the softmax
//                warpgroup of the other tile runs (ping-pong).
//   warps 4-7  : softmax warpgroup of tile 0, warps 8-11: tile 1.  Thread r
//                owns query row r of its tile (TMEM lane r).  Per block it
//                loads the 128 scores of its row, masks boundary blocks, keeps
//                the running max / sum in registers, rescales its O row in
//                TMEM only when the max rose by more than a threshold (the
//                final division uses the same reference, so this is exact),
//                writes P (16-bit, or e4m3 for the FP8 path) into TMEM over
//                the scores, and at the end of the unit normalises O, stores
//                it and the fp32 LSE.
//   TMEM columns: S_0 [0,128) with P_0 at [64,..), S_1 [128,256) with P_1 at
//                [192,..), O_0 [256, 256+D), O_1 [256+D, 256+2D).
//
// Every mbarrier wait is bounded; on a timeout the CTA records the error in
// a device status word, stops issuing work, lets its own copies and MMAs
// drain, frees TMEM and returns.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "sm100.cuh"

namespace fa {

enum : int { DT_FP16 = 0, DT_BF16 = 1, DT_E4M3 = 2 };

// device status word: bit flags of the role whose wait timed out
enum : int {
  ST_TIMEOUT_LOAD = 1,
  ST_TIMEOUT_MMA = 2,
  ST_TIMEOUT_SOFTMAX = 4,
  ST_TIMEOUT_DRAIN = 8,
};

struct FwdParams {
  void* out;           // [B, N_q, H, D] fp16 (fp16 inputs) or bf16
  float* lse;          // [B, H, N_q] fp32, may be null
  int B, Nq, Nk, H;
  int causal;
  int window_left;     // -1 = unlimited
  float score_scale;   // scale * log2(e) * q_descale * k_descale
  float out_scale;     // v_descale (1 for 16-bit inputs)
  int num_units;
  int pairs;           // ceil(N_q / 256)
  unsigned long long wait_limit_ns;
  int* status;         // device status word
};

constexpr int BLOCK_M = 128;   // query rows per tile
constexpr int BLOCK_N = 128;   // keys per block
constexpr int NUM_THREADS = 384;

template <int D, int DT>
struct Cfg {
  static constexpr int ES = DT == DT_E4M3 ? 1 : 2;           // input element bytes
  static constexpr int TILE_BYTES = 128 * D * ES;            // one 128-row tile
  static constexpr int BOX_INNER = 128 / ES;                 // elements per 128-byte row
  static constexpr int NCHUNK = D * ES / 128;                // 128-byte column chunks per row
  static constexpr int CHUNK_BYTES = 128 * 128;              // one chunk of 128 rows
  static constexpr int STAGES = TILE_BYTES >= 32768 ? 4 : 8; // K/V ring slots
  static constexpr int KSTEP = DT == DT_E4M3 ? 32 : 16;      // K per MMA instruction
  static constexpr int P_COLS = 128 * ES / 4;                // TMEM columns of one P row
  static constexpr int P_OFF = 64;                           // P column offset inside S_t
  static constexpr int O_COL0 = 256;
  static constexpr int SMEM_BYTES = 1024 /*barriers*/ + (2 + STAGES) * TILE_BYTES + 1024 /*align*/;
  static constexpr uint32_t FMT = DT == DT_BF16 ? 1u : 0u;
  static constexpr uint32_t IDESC_S = make_idesc(FMT, false, 128, 128);
  static constexpr uint32_t IDESC_O = make_idesc(FMT, true, 128, D);
  // P = 2^PSHIFT * exp2(s - m_used); FP8 shifts P up to use e4m3's range
  static constexpr float PSHIFT = DT == DT_E4M3 ? 7.0f : 0.0f;
  // rescale O only when the row max rose by more than this (log2 units)
  static constexpr float RESCALE_THRESHOLD = DT == DT_E4M3 ? 1.5f : 8.0f;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(D == 64 || D == 128, "head dim");
};

struct SharedHeader {
  uint64_t q_full, q_empty;
  uint64_t kv_full[8], kv_empty[8];
  uint64_t s_full[2], p_full[2], o_full[2], o_empty[2];
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(SharedHeader) <= 1024, "header");

struct Unit {
  int b, h, q0;
  int lo[2], hi[2];
  bool valid[2];   // tile has rows and at least one key block
  bool rows[2];    // tile has rows (< N_q)
  int jlo, jhi;    // union of the valid tiles' block ranges
};

__device__ __forceinline__ Unit get_unit(int u, const FwdParams& p) {
  Unit w;
  const int bh_count = p.B * p.H;
  const int m_idx = u / bh_count;
  // causal: longest units (largest query index) first
  const int m = p.causal ? (p.pairs - 1 - m_idx) : m_idx;
  const int bh = u - m_idx * bh_count;
  w.b = bh / p.H;
  w.h = bh - w.b * p.H;
  w.q0 = m * (2 * BLOCK_M);
  w.jlo = 0x7fffffff;
  w.jhi = -1;
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const int qs = w.q0 + t * BLOCK_M;
    w.rows[t] = qs < p.Nq;
    const int qe = min(qs + BLOCK_M - 1, p.Nq - 1);
    const int lo = p.window_left >= 0 ? max(0, qs - p.window_left) / BLOCK_N : 0;
    const int hi = p.causal ? min(qe, p.Nk - 1) / BLOCK_N : (p.Nk - 1) / BLOCK_N;
    w.lo[t] = lo;
    w.hi[t] = hi;
    w.valid[t] = w.rows[t] && p.Nk > 0 && lo <= hi && (!p.causal || qe >= 0);
    if (w.valid[t]) {
      w.jlo = min(w.jlo, lo);
      w.jhi = max(w.jhi, hi);
    }
  }
  return w;
}

__device__ __forceinline__ void record_error(SharedHeader* sh, const FwdParams& p, int code) {
  atomicOr(p.status, code);
  atomicExch(&sh->abort_flag, 1);
}

__device__ __forceinline__ bool aborted(SharedHeader* sh) {
  return *reinterpret_cast<volatile int*>(&sh->abort_flag) != 0;
}

__device__ __forceinline__ void setmaxnreg_dec80() { asm volatile("setmaxnreg.dec.sync.aligned.u32 80;\n"); }
__device__ __forceinline__ void setmaxnreg_inc208() { asm volatile("setmaxnreg.inc.sync.aligned.u32 208;\n"); }

// ------------------------------------------------------------------ producer
template <int D, int DT>
__device__ void producer_role(SharedHeader* sh, uint8_t* tiles, const CUtensorMap* mq,
                              const CUtensorMap* mk, const CUtensorMap* mv, const FwdParams& p) {
  using C = Cfg<D, DT>;
  uint8_t* sq = tiles;
  uint8_t* ring = tiles + 2 * C::TILE_BYTES;
  uint32_t kv_it = 0;
  uint32_t q_uses = 0;
  uint32_t issued_mask = 0;   // bit s: slot s has had a load
  uint32_t phase_mask = 0;    // bit s: parity of slot s's latest load
  bool q_outstanding = false;
  bool ok = true;
  const uint64_t pol_kv = policy_evict_last();
  const uint64_t pol_q = policy_evict_first();

  for (int u = blockIdx.x; u < p.num_units && ok; u += gridDim.x) {
    const Unit w = get_unit(u, p);
    if (w.jhi < 0) continue;
    if (aborted(sh)) { ok = false; break; }
    // Q tiles (wait until the previous unit's S MMAs have read them)
    if (!mbar_wait(smem_u32(&sh->q_empty), (q_uses & 1u) ^ 1u, p.wait_limit_ns)) {
      record_error(sh, p, ST_TIMEOUT_LOAD); ok = false; break;
    }
    mbar_arrive_expect_tx(smem_u32(&sh->q_full), 2 * C::TILE_BYTES);
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
      for (int c = 0; c < C::NCHUNK; ++c)
        tma_load_4d_hint(smem_u32(sq + t * C::TILE_BYTES + c * C::CHUNK_BYTES), mq, smem_u32(&sh->q_full),
                         c * C::BOX_INNER, w.h, w.q0 + t * BLOCK_M, w.b, pol_q);
    q_outstanding = true;
    ++q_uses;
    // K_j, V_j for the union of the tiles' block ranges
    for (int j = w.jlo; j <= w.jhi && ok; ++j) {
#pragma unroll
      for (int kv = 0; kv < 2; ++kv) {
        const uint32_t slot = kv_it % C::STAGES;
        const uint32_t round = kv_it / C::STAGES;
        if (!mbar_wait(smem_u32(&sh->kv_empty[slot]), (round & 1u) ^ 1u, p.wait_limit_ns)) {
          record_error(sh, p, ST_TIMEOUT_LOAD); ok = false; break;
        }
        const uint32_t bar = smem_u32(&sh->kv_full[slot]);
        mbar_arrive_expect_tx(bar, C::TILE_BYTES);
        const CUtensorMap* map = kv == 0 ? mk : mv;
#pragma unroll
        for (int c = 0; c < C::NCHUNK; ++c)
          tma_load_4d_hint(smem_u32(ring + slot * C::TILE_BYTES + c * C::CHUNK_BYTES), map, bar,
                           c * C::BOX_INNER, w.h, j * BLOCK_N, w.b, pol_kv);
        issued_mask |= 1u << slot;
        phase_mask = (phase_mask & ~(1u << slot)) | ((round & 1u) << slot);
        ++kv_it;
      }
    }
  }
  // drain: every copy this thread issued must land before the CTA exits
  if (!ok) {
#pragma unroll
    for (int s = 0; s < C::STAGES; ++s)
      if (((issued_mask >> s) & 1u) &&
          !mbar_wait(smem_u32(&sh->kv_full[s]), (phase_mask >> s) & 1u, p.wait_limit_ns))
        record_error(sh, p, ST_TIMEOUT_DRAIN);
    if (q_outstanding && !mbar_wait(smem_u32(&sh->q_full), (q_uses - 1u) & 1u, p.wait_limit_ns))
      record_error(sh, p, ST_TIMEOUT_DRAIN);
  }
}

// ------------------------------------------------------------------ MMA issuer
template <int D, int DT>
__device__ __forceinline__ void issue_s(uint32_t d_tmem, uint32_t q_addr, uint32_t k_addr) {
  using C = Cfg<D, DT>;
#pragma unroll
  for (int kk = 0; kk < D / C::KSTEP; ++kk) {
    const int byte = kk * C::KSTEP * C::ES;
    const int off = (byte / 128) * C::CHUNK_BYTES + (byte % 128);
    const uint64_t a = sdesc_sw128(q_addr + off, 16, 1024);
    const uint64_t b = sdesc_sw128(k_addr + off, 16, 1024);
    if constexpr (DT == DT_E4M3) mma_f8_ss(d_tmem, a, b, C::IDESC_S, kk > 0);
    else mma_f16_ss(d_tmem, a, b, C::IDESC_S, kk > 0);
  }
}

template <int D, int DT>
__device__ __forceinline__ void issue_pv(uint32_t d_tmem, uint32_t p_tmem, uint32_t v_addr, bool accumulate) {
  using C = Cfg<D, DT>;
#pragma unroll
  for (int kk = 0; kk < BLOCK_N / C::KSTEP; ++kk) {
    // V tile is MN-major (head dim contiguous): 8-key groups 1024 B apart,
    // 128-byte head-dim chunks CHUNK_BYTES apart.
    const uint64_t b = sdesc_sw128(v_addr + kk * C::KSTEP * 128, C::CHUNK_BYTES, 1024);
    const uint32_t a = p_tmem + kk * (C::KSTEP * C::ES / 4);
    if constexpr (DT == DT_E4M3) mma_f8_ts(d_tmem, a, b, C::IDESC_O, accumulate || kk > 0);
    else mma_f16_ts(d_tmem, a, b, C::IDESC_O, accumulate || kk > 0);
  }
}

template <int D, int DT>
__device__ void mma_role(SharedHeader* sh, uint8_t* tiles, uint32_t tbase, const FwdParams& p) {
  using C = Cfg<D, DT>;
  const uint32_t sq = smem_u32(tiles);
  const uint32_t ring = smem_u32(tiles + 2 * C::TILE_BYTES);
  uint32_t kv_base = 0;
  uint32_t q_uses = 0;
  uint32_t p_waits[2] = {0, 0};
  uint32_t o_units[2] = {0, 0};
  bool ok = true;
  const uint32_t s_tmem[2] = {tbase, tbase + 128};
  const uint32_t p_tmem[2] = {tbase + C::P_OFF, tbase + 128 + C::P_OFF};
  const uint32_t o_tmem[2] = {tbase + C::O_COL0, tbase + C::O_COL0 + D};

  for (int u = blockIdx.x; u < p.num_units && ok; u += gridDim.x) {
    const Unit w = get_unit(u, p);
    if (w.jhi < 0) continue;
    if (aborted(sh)) { ok = false; break; }
    if (!mbar_wait(smem_u32(&sh->q_full), q_uses & 1u, p.wait_limit_ns)) {
      record_error(sh, p, ST_TIMEOUT_MMA); ok = false; break;
    }
    ++q_uses;
    for (int j = w.jlo; j <= w.jhi + 1 && ok; ++j) {
      uint32_t kslot = 0, vslot = 0;
      if (j <= w.jhi) {
        const uint32_t idx = kv_base + 2u * (j - w.jlo);
        kslot = idx % C::STAGES;
        if (!mbar_wait(smem_u32(&sh->kv_full[kslot]), (idx / C::STAGES) & 1u, p.wait_limit_ns)) {
          record_error(sh, p, ST_TIMEOUT_MMA); ok = false; break;
        }
      }
      if (j > w.jlo) {
        const uint32_t idx = kv_base + 2u * (j - 1 - w.jlo) + 1u;
        vslot = idx % C::STAGES;
        if (!mbar_wait(smem_u32(&sh->kv_full[vslot]), (idx / C::STAGES) & 1u, p.wait_limit_ns)) {
          record_error(sh, p, ST_TIMEOUT_MMA); ok = false; break;
        }
      }
      tc_fence_after();
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        if (!w.valid[t]) continue;
        const int jp = j - 1;
        if (jp >= w.lo[t] && jp <= w.hi[t]) {
          // O_t += P_t(j-1) V_{j-1}
          if (!mbar_wait(smem_u32(&sh->p_full[t]), p_waits[t] & 1u, p.wait_limit_ns)) {
            record_error(sh, p, ST_TIMEOUT_MMA); ok = false; break;
          }
          ++p_waits[t];
          if (jp == w.lo[t]) {
            // O_t must have been read out by the previous unit's epilogue
            if (!mbar_wait(smem_u32(&sh->o_empty[t]), (o_units[t] & 1u) ^ 1u, p.wait_limit_ns)) {
              record_error(sh, p, ST_TIMEOUT_MMA); ok = false; break;
            }
          }
          tc_fence_after();
          issue_pv<D, DT>(o_tmem[t], p_tmem[t], ring + vslot * C::TILE_BYTES, jp > w.lo[t]);
          if (jp == w.hi[t]) {
            mma_commit(smem_u32(&sh->o_full[t]));
            ++o_units[t];
          }
        }
        if (j >= w.lo[t] && j <= w.hi[t]) {
          // S_t(j) = Q_t K_j^T   (issued after PV_t(j-1), which read P_t from these columns)
          issue_s<D, DT>(s_tmem[t], sq + t * C::TILE_BYTES, ring + kslot * C::TILE_BYTES);
          mma_commit(smem_u32(&sh->s_full[t]));
        }
      }
      if (!ok) break;
      if (j <= w.jhi) mma_commit(smem_u32(&sh->kv_empty[kslot]));
      if (j > w.jlo) mma_commit(smem_u32(&sh->kv_empty[vslot]));
    }
    if (!ok) break;
    mma_commit(smem_u32(&sh->q_empty));
    kv_base += 2u * (w.jhi - w.jlo + 1);
  }
  // all issued MMAs complete before the CTA releases TMEM
  mma_commit(smem_u32(&sh->mma_done));
  if (!mbar_wait(smem_u32(&sh->mma_done), 0, p.wait_limit_ns)) record_error(sh, p, ST_TIMEOUT_DRAIN);
}

// ------------------------------------------------------------------ softmax
template <int DT>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  if constexpr (DT == DT_FP16) {
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
  } else {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
  }
}

__device__ __forceinline__ uint32_t pack4_e4m3(float a, float b, float c, float d) {
  const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
  const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(make_float2(c, d), __NV_SATFINITE, __NV_E4M3);
  return static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
}

template <int DT>
__device__ __forceinline__ void store_out_row16(void* dst, const float* o, float inv) {
  // 16 values -> two 16-byte stores
  uint4 v0, v1;
  uint32_t* w0 = reinterpret_cast<uint32_t*>(&v0);
  uint32_t* w1 = reinterpret_cast<uint32_t*>(&v1);
  constexpr int OUT_DT = DT == DT_FP16 ? DT_FP16 : DT_BF16;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    w0[i] = pack2<OUT_DT>(o[2 * i] * inv, o[2 * i + 1] * inv);
    w1[i] = pack2<OUT_DT>(o[8 + 2 * i] * inv, o[8 + 2 * i + 1] * inv);
  }
  reinterpret_cast<uint4*>(dst)[0] = v0;
  reinterpret_cast<uint4*>(dst)[1] = v1;
}

template <int D, int DT>
__device__ void softmax_role(SharedHeader* sh, uint32_t tbase, int t, const FwdParams& p) {
  using C = Cfg<D, DT>;
  const int warp_in_wg = (threadIdx.x / 32) & 3;
  const int r = warp_in_wg * 32 + (int)lane_id();      // row in tile == TMEM lane
  const uint32_t lane_off = static_cast<uint32_t>(warp_in_wg * 32) << 16;
  const uint32_t s_col = tbase + lane_off + t * 128;
  const uint32_t p_col = s_col + C::P_OFF;
  const uint32_t o_col = tbase + lane_off + C::O_COL0 + t * D;
  const float cc = p.score_scale;
  uint32_t s_waits = 0, units = 0;
  bool ok = true;
  constexpr int OUT_ES = 2;

  for (int u = blockIdx.x; u < p.num_units && ok; u += gridDim.x) {
    const Unit w = get_unit(u, p);
    if (!w.rows[t]) continue;
    const int row = w.q0 + t * BLOCK_M + r;
    const bool row_ok = row < p.Nq;
    uint8_t* out_row = reinterpret_cast<uint8_t*>(p.out) +
                       ((static_cast<int64_t>(w.b) * p.Nq + row) * p.H + w.h) * (int64_t)D * OUT_ES;
    float* lse_ptr = p.lse ? p.lse + (static_cast<int64_t>(w.b) * p.H + w.h) * p.Nq + row : nullptr;
    if (!w.valid[t]) {
      // no visible key for any row of this tile
      if (row_ok) {
        float z[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) z[i] = 0.f;
#pragma unroll
        for (int c = 0; c < D; c += 16) store_out_row16<DT>(out_row + c * OUT_ES, z, 0.f);
        if (lse_ptr) *lse_ptr = -INFINITY;
      }
      continue;
    }
    if (aborted(sh)) { ok = false; break; }
    float m_used = -INFINITY;   // reference max (log2 units) that P and l are taken against
    float l = 0.f;
    for (int j = w.lo[t]; j <= w.hi[t]; ++j) {
      bool got = mbar_wait(smem_u32(&sh->s_full[t]), s_waits & 1u, p.wait_limit_ns);
      got = __all_sync(0xffffffffu, got);
      if (!got) { record_error(sh, p, ST_TIMEOUT_SOFTMAX); ok = false; break; }
      ++s_waits;
      tc_fence_after();
      float s[BLOCK_N];
      tmem_ld32(s_col + 0, reinterpret_cast<uint32_t*>(s + 0));
      tmem_ld32(s_col + 32, reinterpret_cast<uint32_t*>(s + 32));
      tmem_ld32(s_col + 64, reinterpret_cast<uint32_t*>(s + 64));
      tmem_ld32(s_col + 96, reinterpret_cast<uint32_t*>(s + 96));
      tmem_wait_ld();
      // mask boundary blocks (causal diagonal, window edge, key tail)
      const int k0 = j * BLOCK_N;
      const int qs = w.q0 + t * BLOCK_M;
      const bool need_mask = (k0 + BLOCK_N > p.Nk) || (p.causal && k0 + BLOCK_N - 1 > qs) ||
                             (p.window_left >= 0 && k0 < qs + BLOCK_M - 1 - p.window_left);
      if (need_mask) {
        const int hi_c = min(p.Nk - k0, p.causal ? row - k0 + 1 : BLOCK_N);
        const int lo_c = p.window_left >= 0 ? row - p.window_left - k0 : 0;
#pragma unroll
        for (int c = 0; c < BLOCK_N; ++c)
          if (c < lo_c || c >= hi_c) s[c] = -INFINITY;
      }
      float mx0 = s[0], mx1 = s[1], mx2 = s[2], mx3 = s[3];
#pragma unroll
      for (int c = 4; c < BLOCK_N; c += 4) {
        mx0 = fmaxf(mx0, s[c]);
        mx1 = fmaxf(mx1, s[c + 1]);
        mx2 = fmaxf(mx2, s[c + 2]);
        mx3 = fmaxf(mx3, s[c + 3]);
      }
      const float mx = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3));
      const float m_blk = mx * cc;   // -inf stays -inf (cc > 0)
      const float m_cand = fmaxf(m_used, m_blk);
      const bool need = m_cand > m_used + C::RESCALE_THRESHOLD;
      const bool warp_rescale = __any_sync(0xffffffffu, need);
      // alpha rescales O and l from the old reference to the new one
      float alpha = 1.f;
      if (warp_rescale) {
        alpha = (m_cand == -INFINITY) ? 1.f : ex2_approx(m_used - m_cand);
        m_used = m_cand;
      }
      const float mref = (m_used == -INFINITY) ? 0.f : (m_used - C::PSHIFT);
      const float neg_mref = -mref;
      float l0 = 0.f, l1 = 0.f;
      if constexpr (DT == DT_E4M3) {
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t pw[16];
#pragma unroll
          for (int c = 0; c < 64; c += 4) {
            const int cb = half * 64 + c;
            const float e0 = ex2_approx(fmaf(s[cb], cc, neg_mref));
            const float e1 = ex2_approx(fmaf(s[cb + 1], cc, neg_mref));
            const float e2 = ex2_approx(fmaf(s[cb + 2], cc, neg_mref));
            const float e3 = ex2_approx(fmaf(s[cb + 3], cc, neg_mref));
            l0 += e0 + e1;
            l1 += e2 + e3;
            pw[c / 4] = pack4_e4m3(e0, e1, e2, e3);
          }
          tmem_st16(p_col + half * 16, pw);
        }
      } else {
#pragma unroll
        for (int quarter = 0; quarter < 4; ++quarter) {
          uint32_t pw[16];
#pragma unroll
          for (int c = 0; c < 32; c += 2) {
            const float e0 = ex2_approx(fmaf(s[quarter * 32 + c], cc, neg_mref));
            const float e1 = ex2_approx(fmaf(s[quarter * 32 + c + 1], cc, neg_mref));
            l0 += e0;
            l1 += e1;
            pw[c / 2] = pack2<DT>(e0, e1);
          }
          tmem_st16(p_col + quarter * 16, pw);
        }
      }
      // O rescale (only when some row of this warp raised its reference);
      // PV_t(j-1) has completed: S_t(j) was issued after it and has landed.
      if (warp_rescale && j > w.lo[t]) {
#pragma unroll
        for (int c = 0; c < D; c += 16) {
          uint32_t o[16];
          tmem_ld16(o_col + c, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st16(o_col + c, o);
        }
      }
      l = l * alpha;
      l += l0 + l1;
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(smem_u32(&sh->p_full[t]));
    }
    if (!ok) break;
    // epilogue: O / l, LSE
    bool got = mbar_wait(smem_u32(&sh->o_full[t]), units & 1u, p.wait_limit_ns);
    got = __all_sync(0xffffffffu, got);
    if (!got) { record_error(sh, p, ST_TIMEOUT_SOFTMAX); ok = false; break; }
    ++units;
    tc_fence_after();
    const float inv = (l > 0.f ? 1.f / l : 0.f) * p.out_scale;
#pragma unroll
    for (int c = 0; c < D; c += 32) {
      uint32_t o[32];
      tmem_ld32(o_col + c, o);
      tmem_wait_ld();
      if (row_ok) {
        store_out_row16<DT>(out_row + c * OUT_ES, reinterpret_cast<float*>(o), inv);
        store_out_row16<DT>(out_row + (c + 16) * OUT_ES, reinterpret_cast<float*>(o) + 16, inv);
      }
    }
    tc_fence_before();
    mbar_arrive(smem_u32(&sh->o_empty[t]));
    if (row_ok && lse_ptr) {
      // natural log of sum_j exp(scale * s_j) = (m_used + log2(l) - PSHIFT) * ln 2
      *lse_ptr = l > 0.f ? (m_used + __log2f(l) - C::PSHIFT) * 0.69314718055994531f : -INFINITY;
    }
  }
}

// ------------------------------------------------------------------ kernel
template <int D, int DT>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using C = Cfg<D, DT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  SharedHeader* sh = reinterpret_cast<SharedHeader*>(smem);
  uint8_t* tiles = smem + 1024;
  const int warp = threadIdx.x / 32;

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&sh->q_full), 1);
    mbar_init(smem_u32(&sh->q_empty), 1);
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(smem_u32(&sh->kv_full[s]), 1);
      mbar_init(smem_u32(&sh->kv_empty[s]), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(smem_u32(&sh->s_full[t]), 1);
      mbar_init(smem_u32(&sh->p_full[t]), 128);
      mbar_init(smem_u32(&sh->o_full[t]), 1);
      mbar_init(smem_u32(&sh->o_empty[t]), 128);
    }
    mbar_init(smem_u32(&sh->mma_done), 1);
    sh->abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_map(&tm_q);
    tma_prefetch_map(&tm_k);
    tma_prefetch_map(&tm_v);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&sh->tmem_base), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = sh->tmem_base;

  if (warp < 4) {
    setmaxnreg_dec80();
    if (warp == 0 && lane_id() == 0) producer_role<D, DT>(sh, tiles, &tm_q, &tm_k, &tm_v, p);
    else if (warp == 1 && lane_id() == 0) mma_role<D, DT>(sh, tiles, tbase, p);
  } else {
    setmaxnreg_inc208();
    softmax_role<D, DT>(sh, tbase, warp < 8 ? 0 : 1, p);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

// Rows of a problem with N_k = 0 see no key: O = 0, LSE = -inf.
template <int D, int OUT_ES>
__global__ void fa_empty_kernel(void* out, float* lse, int B, int Nq, int H) {
  const int64_t rows = static_cast<int64_t>(B) * Nq * H;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < rows; i += (int64_t)gridDim.x * blockDim.x) {
    uint4* o = reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(out) + i * D * OUT_ES);
#pragma unroll
    for (int c = 0; c < D * OUT_ES / 16; ++c) o[c] = make_uint4(0, 0, 0, 0);
    if (lse) {
      // i enumerates (b, n, h); LSE is [B, H, N_q]
      const int64_t h = i % H;
      const int64_t bn = i / H;
      const int64_t n = bn % Nq;
      const int64_t b = bn / Nq;
      lse[(b * H + h) * Nq + n] = -INFINITY;
    }
  }
}

// A wait that nothing completes: checks that the bounded wait returns.
__global__ void fa_wait_probe_kernel(unsigned long long limit_ns, int* status) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (!mbar_wait(smem_u32(&bar), 0, limit_ns)) atomicOr(status, ST_TIMEOUT_SOFTMAX);
  __syncthreads();
}

}  // namespace fa
