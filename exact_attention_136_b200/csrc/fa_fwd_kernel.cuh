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
//   warps 4-11 : softmax of tile 0 (two warpgroups), warps 12-19: tile 1.
//                Two threads per query row: the tcgen05 16x32bx2 access gives
//                lanes t and t+16 of a warp the two 64-key halves of one TMEM
//                lane (= row), so a row max or sum is one shuffle.  Per block
//                they load the row's 128 scores, mask boundary blocks, keep
//                the running max / sum in registers, rescale the O row in
//                TMEM only when the max rose by more than a threshold (the
//                final division uses the same reference, so this is exact),
//                write P (16-bit, or e4m3 for the FP8 path) into TMEM over
//                the scores, and at the end of the unit normalise O and store
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

// kernel instantiations with a mask on the scores or the probabilities:
// an attention mask (boolean, additive) or dropout of the probabilities
enum : int { MASK_NONE = 0, MASK_BOOL = 1, MASK_ADD = 2, MASK_DROPOUT = 3 };

// device status word: bit flags of the role whose wait timed out
enum : int {
  ST_TIMEOUT_LOAD = 1,
  ST_TIMEOUT_MMA = 2,
  ST_TIMEOUT_SOFTMAX = 4,
  ST_TIMEOUT_DRAIN = 8,
  ST_SMEM_MISALIGNED = 16,
};

// Philox4x32-10 round keys: round r uses (seed_lo + r * 0x9E3779B9,
// seed_hi + r * 0xBB67AE85) mod 2^32.  Computed once on the host and read
// from the kernel parameters, so a round costs two wide multiplies and two
// three-input XORs.
struct PhiloxKeys {
  unsigned k0[10], k1[10];
};

inline PhiloxKeys philox_round_keys(unsigned seed_lo, unsigned seed_hi) {
  PhiloxKeys k;
  for (int r = 0; r < 10; ++r) {
    k.k0[r] = seed_lo + static_cast<unsigned>(r) * 0x9E3779B9u;
    k.k1[r] = seed_hi + static_cast<unsigned>(r) * 0xBB67AE85u;
  }
  return k;
}

struct FwdParams {
  void* out;           // [B, N_q, H, D] fp16 (fp16 inputs) or bf16
  float* lse;          // [B, H, N_q] fp32, may be null
  int B, Nq, Nk, H;
  int Hkv;             // key/value heads (H a multiple of Hkv)
  int qpk;             // H / Hkv: query head h reads K/V head h / qpk
  int causal;          // scheduling order only; the key bounds below carry the mask
  int window_left;     // keys at most this many before the query; -1 = unlimited
  int window_right;    // keys at most this many after the query; -1 = unlimited,
                       // 0 under causal (set by the host, below N_k + N_q < 2^31)
  float score_scale;   // scale * log2(e) * q_descale * k_descale
  float out_scale;     // v_descale (1 for 16-bit inputs)
  int num_units;
  int pairs;           // ceil(N_q / 256): work units per (batch, head)
  int group;           // (batch, head) pairs per scheduling group (see get_tile)
  unsigned* sched;     // [2] scheduler scratch: next unit to claim, CTAs finished;
                       // zero between launches (the last CTA resets it)
  unsigned long long wait_limit_ns;
  int* status;         // device status word
  // split key range (decode-like shapes): every work unit covers key blocks
  // [s * split_blocks, (s + 1) * split_blocks) of one slice s and writes its
  // O (normalised by the slice's own row sum) and LSE in fp32 to the
  // partial buffers; a merge kernel combines the slices.  splits = 1: O and
  // LSE go straight to out / lse.
  int splits;
  int split_blocks;
  float* o_part;       // [splits, B, N_q, H, D]
  float* lse_part;     // [splits, B, H, N_q]
  // attention mask (masked kernels): element (b, h, i, j) at
  // mask + b * mask_sb + h * mask_sh + i * mask_sq + j; boolean masks are
  // bytes (0 = masked out), additive ones 16-bit floats added to the scaled
  // score, applied to the raw score as mask * mask_scale
  const void* mask;
  long long mask_sb, mask_sh, mask_sq;
  float mask_scale;    // 1 / (scale * q_descale * k_descale)
  // dropout (MASK_DROPOUT kernels): key j of row i of (batch b, query head
  // h) is kept when a 16-bit value of Philox4x32-10 at counter
  // (j / 8, i, b * H + h, drop_offset) under key (seed_lo, seed_hi) is at
  // least drop_threshold; out_scale already holds the 1 / (1 - p)
  unsigned drop_threshold;
  unsigned seed_lo, seed_hi, drop_offset;
  PhiloxKeys drop_keys;   // the round keys of (seed_lo, seed_hi)
  // packed variable-length batches (cu_q non-null): sequence b holds query
  // rows [cu_q[b], cu_q[b+1]) of q / out ([total_q, H, D]) and keys
  // [cu_k[b], cu_k[b+1]) of k / v ([total_k, H_kv, D]); LSE is [H, total_q];
  // N_q is then the longest sequence (it sizes the work units)
  const int* cu_q;
  const int* cu_k;
  int total_q, total_k;
};

// Exponentials taken on the FMA pipe (see Cfg::EMU_FROM): pairs i >= this of
// every 8, per instantiation; 8 = none.
#ifndef FA_EMU_FROM_D128
#define FA_EMU_FROM_D128 8
#endif
#ifndef FA_EMU_FROM_D64
#define FA_EMU_FROM_D64 8
#endif
#ifndef FA_EMU_FROM_E4M3
#define FA_EMU_FROM_E4M3 8
#endif

constexpr int BLOCK_M = 128;   // query rows per tile
constexpr int BLOCK_N = 128;   // keys per block
constexpr int NUM_THREADS = 640;   // warpgroup 0: load + MMA; 2 warpgroups per Q tile
constexpr int HEADER_BYTES = 1024;  // mbarriers and flags
constexpr int XCH_BYTES = 0;        // (no shared-memory exchange)

template <int D, int DT, int MASK = 0>
struct Cfg {
  static constexpr int ES = DT == DT_E4M3 ? 1 : 2;           // input element bytes
  static constexpr int TILE_BYTES = 128 * D * ES;            // one 128-row tile
  static constexpr int BOX_INNER = 128 / ES;                 // elements per 128-byte row
  static constexpr int NCHUNK = D * ES / 128;                // 128-byte column chunks per row
  static constexpr int CHUNK_BYTES = 128 * 128;              // one chunk of 128 rows
  // Attention-mask tiles (boolean: 1 byte, additive: 2 bytes per element)
  // staged by TMA: per Q tile, M_SLOTS slots of 128 rows x 128 keys
  static constexpr bool TMA_MASK = MASK == MASK_BOOL || MASK == MASK_ADD;
  static constexpr int MES = MASK == MASK_BOOL ? 1 : 2;
  static constexpr int M_TILE = 128 * 128 * MES;
  static constexpr int M_SLOTS = MASK == MASK_BOOL ? 2 : (MASK == MASK_ADD ? 1 : 0);
  static constexpr int M_BYTES = 2 * M_SLOTS * M_TILE;
  // K/V ring slots: whatever shared memory is left after the header, the
  // exchange buffer, Q0, Q1 and the mask slots
  static constexpr int STAGES_FIT = (232448 - HEADER_BYTES - XCH_BYTES - 2 * TILE_BYTES - M_BYTES) / TILE_BYTES;
  static constexpr int STAGES = STAGES_FIT > 12 ? 12 : STAGES_FIT;
  static constexpr int OFF_MASK = (2 + STAGES) * TILE_BYTES;   // from the first Q tile
  static constexpr int KSTEP = DT == DT_E4M3 ? 32 : 16;      // K per MMA instruction
  static constexpr int P_COLS = 128 * ES / 4;                // TMEM columns of one P row
  static constexpr int P_OFF = 64;                           // P column offset inside S_t
  static constexpr int O_COL0 = 256;
  // the dynamic shared memory base is 1024-byte aligned (checked at entry)
  static constexpr int SMEM_BYTES = HEADER_BYTES + XCH_BYTES + (2 + STAGES) * TILE_BYTES + M_BYTES;
  static constexpr uint32_t FMT = DT == DT_BF16 ? 1u : 0u;
  static constexpr uint32_t IDESC_S = make_idesc(FMT, false, 128, 128);
  static constexpr uint32_t IDESC_O = make_idesc(FMT, true, 128, D);
  // P = 2^PSHIFT * exp2(s - m_used); FP8 shifts P up to use e4m3's range
  static constexpr float PSHIFT = DT == DT_E4M3 ? 7.0f : 0.0f;
  // rescale O only when the row max rose by more than this (log2 units)
  static constexpr float RESCALE_THRESHOLD = DT == DT_E4M3 ? 1.5f : 8.0f;
  // P is handed to the MMA thread in two halves (keys k with k mod 64 below
  // 32 first), so the first PV MMAs run while the rest is exponentiated.
  // Measured on B200: faster for 16-bit inputs; for e4m3, whose PV is only
  // four MMAs, the extra hand-over costs more than the overlap gains.
  static constexpr bool PSPLIT = DT != DT_E4M3;
  // Exponentials on the FMA pipe: pairs i >= EMU_FROM of every 8 in a block
  // without masked keys take exp2_poly instead of MUFU (8 = none), with a
  // polynomial of degree EMU_DEG (P is rounded to e4m3's 3-bit mantissa in
  // the FP8 path, so degree 2 is ample there).
  static constexpr int EMU_FROM = DT == DT_E4M3 ? FA_EMU_FROM_E4M3 : (D == 64 ? FA_EMU_FROM_D64 : FA_EMU_FROM_D128);
  static constexpr int EMU_DEG = DT == DT_E4M3 ? 2 : 3;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(STAGES >= 3, "K/V ring");
  static_assert(D == 64 || D == 128, "head dim");
};

struct SharedHeader {
  uint64_t q_full[2], q_empty[2];   // per Q tile: loaded / read by the tile's last S
  uint64_t kv_full[12], kv_empty[12];
  uint64_t s_full[2], p_full[2], o_full[2], o_empty[2];
  uint64_t p_half[2];   // first half of P_t stored (keys k of the block with k mod 64 < 32)
  uint64_t m_full[2][2], m_empty[2][2];   // attention-mask slots per Q tile: loaded / read
  uint64_t mma_done;
  uint64_t uq_full[4], uq_empty[4];   // unit queue: producer -> MMA + softmax warps
  int uq[4];                          // claimed unit ids, -1 = no more work
  int uq_split[4];                    // ... and their key-range slices
  uint32_t tmem_base;
  int abort_flag;
#ifdef FA_STATS_BUILD
  unsigned stats[64];
#endif
};
static_assert(sizeof(SharedHeader) <= HEADER_BYTES, "header");

// One 128-row query tile of a work unit and its key-block range.
struct Tile {
  int b, h, qs;    // batch (sequence), head, first query row (within the sequence)
  int hk;          // key/value head of this query head
  int lo, hi;      // inclusive key-block range
  int split;       // key-range slice (0 when not split)
  bool rows;       // tile has rows (qs < nq)
  bool valid;      // ... and at least one key block
  int nq, nk;      // the sequence's query rows and keys
  int qrow0, krow0, tb;   // TMA row of its first query / key, and TMA batch coordinate
  int64_t orow0;   // out row (of [rows, H, D]) of its first query
  int64_t lse0;    // LSE element of its first query
};

// Work-unit order.  Units are numbered group by group, a group being
// `p.group` consecutive (batch, head) pairs whose K and V fit in L2 together;
// inside a group causal units run longest first (largest query index), and
// consecutive units switch head so the CTAs working at the same time share
// each head's K/V blocks through L2.  Non-causal units use groups of one head.
template <bool SPLIT>
__device__ __forceinline__ Tile get_tile(int u, int split, int t, const FwdParams& p) {
  Tile w;
  w.split = split;
  const int bh_count = p.B * p.H;
  const int per_group = p.group * p.pairs;
  const int g = u / per_group;
  const int r = u - g * per_group;
  const int g_heads = min(p.group, bh_count - g * p.group);
  const int m_idx = r / g_heads;
  const int bh = g * p.group + (r - m_idx * g_heads);
  const int m = p.causal ? (p.pairs - 1 - m_idx) : m_idx;
  w.b = bh / p.H;
  w.h = bh - w.b * p.H;
  w.hk = w.h / p.qpk;
  w.qs = m * (2 * BLOCK_M) + t * BLOCK_M;
  if (p.cu_q) {
    // a packed sequence: its rows and keys, clamped into the packed tensors
    const int q_start = min(max(__ldg(p.cu_q + w.b), 0), p.total_q);
    const int k_start = min(max(__ldg(p.cu_k + w.b), 0), p.total_k);
    w.nq = min(max(__ldg(p.cu_q + w.b + 1), q_start), p.total_q) - q_start;
    w.nk = min(max(__ldg(p.cu_k + w.b + 1), k_start), p.total_k) - k_start;
    w.qrow0 = q_start;
    w.krow0 = k_start;
    w.tb = 0;
    w.orow0 = q_start;
    w.lse0 = static_cast<int64_t>(w.h) * p.total_q + q_start;
  } else {
    w.nq = p.Nq;
    w.nk = p.Nk;
    w.qrow0 = 0;
    w.krow0 = 0;
    w.tb = w.b;
    w.orow0 = static_cast<int64_t>(w.b) * p.Nq;
    w.lse0 = (static_cast<int64_t>(w.b) * p.H + w.h) * p.Nq;
  }
  w.rows = w.qs < w.nq;
  const int qe = min(w.qs + BLOCK_M - 1, w.nq - 1);
  w.lo = p.window_left >= 0 ? max(0, w.qs - p.window_left) / BLOCK_N : 0;
  w.hi = p.window_right >= 0 ? min(qe + p.window_right, w.nk - 1) / BLOCK_N : (w.nk - 1) / BLOCK_N;
  if (SPLIT) {
    w.lo = max(w.lo, w.split * p.split_blocks);
    w.hi = min(w.hi, (w.split + 1) * p.split_blocks - 1);
  }
  w.valid = w.rows && w.nk > 0 && w.lo <= w.hi;
  return w;
}

// Both tiles of a work unit and the union of their key-block ranges.
struct Unit {
  int b, h, hk, q0;
  int qrow0, krow0, tb;   // TMA row of the sequence's first query / key, TMA batch coordinate
  int lo[2], hi[2];
  bool valid[2];
  int jlo, jhi;    // empty (jhi < 0) when neither tile has work
};

template <bool SPLIT>
__device__ __forceinline__ Unit get_unit(int u, int split, const FwdParams& p) {
  const Tile a = get_tile<SPLIT>(u, split, 0, p);
  const Tile c = get_tile<SPLIT>(u, split, 1, p);
  Unit w;
  w.b = a.b;
  w.h = a.h;
  w.hk = a.hk;
  w.q0 = a.qs;
  w.qrow0 = a.qrow0;
  w.krow0 = a.krow0;
  w.tb = a.tb;
  w.lo[0] = a.lo; w.hi[0] = a.hi; w.valid[0] = a.valid;
  w.lo[1] = c.lo; w.hi[1] = c.hi; w.valid[1] = c.valid;
  w.jlo = a.valid ? a.lo : (c.valid ? c.lo : 0);
  if (a.valid && c.valid) w.jlo = min(a.lo, c.lo);
  w.jhi = a.valid ? a.hi : -1;
  if (c.valid) w.jhi = max(w.jhi, c.hi);
  return w;
}

// Optional event tracing for timeline studies (off in the library build):
// lane 0 of one warp per role in CTA 0 stores (event, block, clock) records
// into its own slice of g_trace with a register counter (no atomics, so the
// tracer adds no round trip to the traced path).
#ifdef FA_TRACE_BUILD
__device__ unsigned long long* g_trace;
constexpr int kTraceSlice = 16384;
#define FA_TRACE_DECL                                                                                 \
  unsigned trace_n = 0;                                                                               \
  unsigned long long* const trace_p = blockIdx.x == 0 ? g_trace : nullptr
#define FA_TRACE(who, ev, j)                                                                          \
  do {                                                                                                \
    if (trace_p && ((who) >= 2 || threadIdx.x == 128u + 256u * (who)) && trace_n < kTraceSlice)       \
      trace_p[(who) * kTraceSlice + trace_n++] =                                                      \
          (static_cast<unsigned long long>((ev) & 0xff) << 48) |                                     \
          (static_cast<unsigned long long>((j) & 0xffff) << 32) |                                    \
          (static_cast<unsigned long long>(clock64()) & 0xffffffffull);                              \
  } while (0)
#elif defined(FA_STATS_BUILD)
// Tuning build: the time between consecutive events of a role is summed per
// (role, event) in shared memory by the role's recording thread (lane 0 of
// one warp per role and softmax warpgroup) and added to g_stats at exit.
__device__ unsigned long long g_stats[64];
#define FA_TRACE_DECL uint32_t stat_last = static_cast<uint32_t>(clock())
#define FA_TRACE(who, ev, j)                                                      \
  do {                                                                            \
    if ((who) >= 2 || (threadIdx.x & 127) == 0) {                                 \
      const uint32_t now_ = static_cast<uint32_t>(clock());                       \
      atomicAdd(&sh->stats[(who) * 16 + (ev)], now_ - stat_last);                 \
      stat_last = now_;                                                           \
    }                                                                             \
  } while (0)
#else
#define FA_TRACE_DECL do { } while (0)
#define FA_TRACE(who, ev, j) do { } while (0)
#endif

// Dynamic schedule: CTAs claim units in order from a global counter, so the
// units running at any time are a contiguous stretch of the longest-first,
// head-grouped order (balanced and L2-friendly).  The producer thread claims
// and passes each unit to the MMA thread and the softmax warps through a
// 4-deep queue in shared memory.
constexpr uint32_t UQ_CONSUMERS = 1 + 16;   // MMA thread + one arrive per softmax warp

// Units [0, gridDim.x) are each CTA's first unit (no atomic on the start-up
// path); later units come from the counter.
__device__ __forceinline__ int claim_unit(const FwdParams& p) {
  const int u = static_cast<int>(gridDim.x + atomicAdd(p.sched, 1u));
  return u < p.num_units ? u : -1;
}

__device__ __forceinline__ void record_error(SharedHeader* sh, const FwdParams& p, int code) {
  atomicOr(p.status, code);
  atomicExch(&sh->abort_flag, 1);
}

__device__ __forceinline__ bool aborted(SharedHeader* sh) {
  return *reinterpret_cast<volatile int*>(&sh->abort_flag) != 0;
}

// Register split between warpgroup 0 (one producer and one MMA thread) and
// the four softmax warpgroups.  The launch gives every thread 96 registers
// (640 threads, one CTA per SM: 61440 of the SM's 65536; the kernel is
// compiled to exactly that, checked by the host before the first launch);
// the split must not exceed that total.
constexpr int REGS_LAUNCH = 96;
constexpr int REGS_LOAD_MMA = 64;
constexpr int REGS_SOFTMAX = 104;
static_assert(NUM_THREADS * REGS_LAUNCH <= 65536, "launch registers");
static_assert(128 * REGS_LOAD_MMA + 512 * REGS_SOFTMAX <= NUM_THREADS * REGS_LAUNCH, "register split");
template <int N>
__device__ __forceinline__ void setmaxnreg_dec() { asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(N)); }
template <int N>
__device__ __forceinline__ void setmaxnreg_inc() { asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(N)); }

// ------------------------------------------------------------------ producer
template <int D, int DT, bool SPLIT, int MASK>
__device__ void producer_role(SharedHeader* sh, uint8_t* tiles, const CUtensorMap* mq,
                              const CUtensorMap* mk, const CUtensorMap* mv, const CUtensorMap* mm,
                              const FwdParams& p) {
  using C = Cfg<D, DT, MASK>;
  uint8_t* sq = tiles;
  uint8_t* ring = tiles + 2 * C::TILE_BYTES;
  uint32_t kv_it = 0;
  uint32_t m_it[2] = {0u, 0u};   // mask tiles loaded per Q tile
  uint32_t m_issued = 0;         // bit 2t + s: mask slot s of tile t has had a load
  uint32_t m_phase = 0;          // ... and the parity of its latest
  uint32_t q_uses = 0;
  uint32_t issued_mask = 0;   // bit s: slot s has had a load
  uint32_t phase_mask = 0;    // bit s: parity of slot s's latest load
  uint32_t q_loaded = 0;       // bit t: Q tile t has had a load
  uint32_t q_phase = 0;        // bit t: parity of Q tile t's latest load
  bool ok = true;
  FA_TRACE_DECL;
  const uint64_t pol_kv = policy_evict_last();
  const uint64_t pol_q = policy_evict_first();

  int k = 0;
  int cur = static_cast<int>(blockIdx.x);   // grid <= num_units
  while (true) {
    // publish the unit to the consumers (-1 ends their loops)
    const uint32_t qs = k & 3u, qr = static_cast<uint32_t>(k) >> 2;
    if (!mbar_wait(smem_u32(&sh->uq_empty[qs]), (qr & 1u) ^ 1u, p.wait_limit_ns)) {
      record_error(sh, p, ST_TIMEOUT_LOAD); ok = false; break;
    }
    // a claimed index enumerates (unit, slice) with the slices of a unit
    // consecutive; decoded once here for every role
    const int cu = (cur < 0 || !SPLIT) ? cur : cur / p.splits;
    const int cs = (cur < 0 || !SPLIT) ? 0 : cur - cu * p.splits;
    sh->uq[qs] = cu;
    sh->uq_split[qs] = cs;
    mbar_arrive(smem_u32(&sh->uq_full[qs]));
    ++k;
    if (cur < 0) break;
    const Unit w = get_unit<SPLIT>(cu, cs, p);
    int nxt = -2;   // claimed once this unit's first loads are on their way
    if (w.jhi < 0) {
      cur = claim_unit(p);
      continue;
    }
    if (aborted(sh)) { ok = false; break; }
    // Q tiles, each as soon as the previous unit's last S of that tile has
    // read it (tile 0's last S of a causal unit comes a key block before
    // tile 1's, so its next Q loads during the unit's last block)
#pragma unroll
    for (int t = 0; t < 2 && ok; ++t) {
      if (!mbar_wait(smem_u32(&sh->q_empty[t]), (q_uses & 1u) ^ 1u, p.wait_limit_ns)) {
        record_error(sh, p, ST_TIMEOUT_LOAD); ok = false; break;
      }
      mbar_arrive_expect_tx(smem_u32(&sh->q_full[t]), C::TILE_BYTES);
#pragma unroll
      for (int c = 0; c < C::NCHUNK; ++c)
        tma_load_4d_hint(smem_u32(sq + t * C::TILE_BYTES + c * C::CHUNK_BYTES), mq, smem_u32(&sh->q_full[t]),
                         c * C::BOX_INNER, w.h, w.qrow0 + w.q0 + t * BLOCK_M, w.tb, pol_q);
      q_loaded |= 1u << t;
      q_phase = (q_phase & ~(1u << t)) | ((q_uses & 1u) << t);
    }
    if (!ok) break;
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
        FA_TRACE(3, 1 + kv, j);
        const uint32_t bar = smem_u32(&sh->kv_full[slot]);
        mbar_arrive_expect_tx(bar, C::TILE_BYTES);
        const CUtensorMap* map = kv == 0 ? mk : mv;
#pragma unroll
        for (int c = 0; c < C::NCHUNK; ++c)
          tma_load_4d_hint(smem_u32(ring + slot * C::TILE_BYTES + c * C::CHUNK_BYTES), map, bar,
                           c * C::BOX_INNER, w.hk, w.krow0 + j * BLOCK_N, w.tb, pol_kv);
        issued_mask |= 1u << slot;
        phase_mask = (phase_mask & ~(1u << slot)) | ((round & 1u) << slot);
        ++kv_it;
      }
      if constexpr (C::TMA_MASK) {
        // this block's mask tile of each Q tile that computes the block
        // (rows past N_q and keys past N_k read as zero)
        const int mh = p.mask_sh != 0 ? w.h : 0, mb = p.mask_sb != 0 ? w.b : 0;
#pragma unroll
        for (int t = 0; t < 2 && ok; ++t) {
          if (!w.valid[t] || j < w.lo[t] || j > w.hi[t]) continue;
          const uint32_t ms = m_it[t] % C::M_SLOTS, mr = m_it[t] / C::M_SLOTS;
          if (!mbar_wait(smem_u32(&sh->m_empty[t][ms]), (mr & 1u) ^ 1u, p.wait_limit_ns)) {
            record_error(sh, p, ST_TIMEOUT_LOAD); ok = false; break;
          }
          const uint32_t bar = smem_u32(&sh->m_full[t][ms]);
          mbar_arrive_expect_tx(bar, C::M_TILE);
          uint8_t* dst = tiles + C::OFF_MASK + (t * C::M_SLOTS + ms) * C::M_TILE;
#pragma unroll
          for (int c = 0; c < C::MES; ++c)   // 128-byte column chunks of 128 rows
            tma_load_4d(smem_u32(dst + c * C::CHUNK_BYTES), mm, bar, j * BLOCK_N + c * (128 / C::MES),
                        w.q0 + t * BLOCK_M, mh, mb);
          m_issued |= 1u << (2 * t + ms);
          m_phase = (m_phase & ~(1u << (2 * t + ms))) | ((mr & 1u) << (2 * t + ms));
          ++m_it[t];
        }
      }
      if (nxt == -2) {
        // claim the next unit while these loads are in flight, and warm L2
        // with its Q tiles
        nxt = claim_unit(p);
        if (nxt >= 0) {
          const int nu = SPLIT ? nxt / p.splits : nxt;
          const Unit wn = get_unit<SPLIT>(nu, SPLIT ? nxt - nu * p.splits : 0, p);
#pragma unroll
          for (int t = 0; t < 2; ++t)
#pragma unroll
            for (int c = 0; c < C::NCHUNK; ++c)
              tma_prefetch_l2_4d(mq, c * C::BOX_INNER, wn.h, wn.qrow0 + wn.q0 + t * BLOCK_M, wn.tb);
        }
      }
    }
    if (!ok) break;
    cur = nxt;
  }
  // drain: every copy this thread issued must land before the CTA exits
  if (!ok) {
#pragma unroll
    for (int s = 0; s < C::STAGES; ++s)
      if (((issued_mask >> s) & 1u) &&
          !mbar_wait(smem_u32(&sh->kv_full[s]), (phase_mask >> s) & 1u, p.wait_limit_ns))
        record_error(sh, p, ST_TIMEOUT_DRAIN);
#pragma unroll
    for (int t = 0; t < 2; ++t)
      if (((q_loaded >> t) & 1u) && !mbar_wait(smem_u32(&sh->q_full[t]), (q_phase >> t) & 1u, p.wait_limit_ns))
        record_error(sh, p, ST_TIMEOUT_DRAIN);
    if constexpr (C::TMA_MASK) {
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (((m_issued >> i) & 1u) &&
            !mbar_wait(smem_u32(&sh->m_full[i / 2][i % 2]), (m_phase >> i) & 1u, p.wait_limit_ns))
          record_error(sh, p, ST_TIMEOUT_DRAIN);
    }
  }
  FA_TRACE(3, 15, 0);
}

// ------------------------------------------------------------------ MMA issuer
// Opaque copy: keeps the compiler from hoisting per-iteration descriptor math
// out of the key-block loop, which would hold dozens of descriptors in
// registers.
__device__ __forceinline__ uint32_t opaque(uint32_t x) {
  asm volatile("mov.b32 %0, %0;" : "+r"(x));
  return x;
}

// Every shared-memory descriptor here has the same high word: 8-row groups
// 1024 B apart (stride byte offset), descriptor version 1, 128-byte swizzle.
constexpr uint32_t DESC_HI = sdesc_sw128_hi(1024);

// S = Q K^T for one 128-row tile.  a0 / b0 are the descriptor low words of
// the K-major 128B-swizzled Q and K tiles; the K step advances 32 B inside a
// 128-byte row, then jumps to the next 128-byte column chunk.
template <int D, int DT>
__device__ __forceinline__ void issue_s(uint32_t d_tmem, uint32_t a0, uint32_t b0, uint32_t hi) {
  using C = Cfg<D, DT>;
#pragma unroll
  for (int kk = 0; kk < D / C::KSTEP; ++kk) {
    const int byte = kk * C::KSTEP * C::ES;
    const uint32_t off = static_cast<uint32_t>(((byte / 128) * C::CHUNK_BYTES + (byte % 128)) >> 4);
    if constexpr (DT == DT_E4M3) mma_f8_ss_lo(d_tmem, a0 + off, b0 + off, hi, C::IDESC_S, kk > 0);
    else mma_f16_ss_lo(d_tmem, a0 + off, b0 + off, hi, C::IDESC_S, kk > 0);
  }
}

// O += P V with P read from TMEM.  b0 is the descriptor low word of the
// MN-major V tile (head dim contiguous): 8-key groups 1024 B apart, 128-byte
// head-dim chunks CHUNK_BYTES apart (the leading byte offset).
// PART 0 / 1 issue only the MMAs over keys k with k mod 64 below / at or
// above 32 (the two halves in which the softmax hands P over: each thread
// holds 64 keys of a row and exponentiates them in order), PART 2 all.
template <int D, int DT, int PART = 2>
__device__ __forceinline__ void issue_pv(uint32_t d_tmem, uint32_t p_tmem, uint32_t b0, uint32_t hi,
                                         bool accumulate) {
  using C = Cfg<D, DT>;
#pragma unroll
  for (int kk = 0; kk < BLOCK_N / C::KSTEP; ++kk) {
    const bool first_half = (kk * C::KSTEP) % 64 < 32;
    if ((PART == 0 && !first_half) || (PART == 1 && first_half)) continue;
    const uint32_t off = static_cast<uint32_t>((kk * C::KSTEP * 128) >> 4);
    const uint32_t a = p_tmem + kk * (C::KSTEP * C::ES / 4);
    if constexpr (DT == DT_E4M3) mma_f8_ts_lo(d_tmem, a, b0 + off, hi, C::IDESC_O, accumulate || kk > 0);
    else mma_f16_ts_lo(d_tmem, a, b0 + off, hi, C::IDESC_O, accumulate || kk > 0);
  }
}

// Ring position (slot, phase parity) of the next load.
template <int STAGES>
__device__ __forceinline__ void ring_next(uint32_t& slot, uint32_t& par) {
  ++slot;
  if (slot == static_cast<uint32_t>(STAGES)) {
    slot = 0;
    par ^= 1u;
  }
}

// O_t += P_t V for one key block, issued as the softmax hands P over: with
// the split hand-over (Cfg::PSPLIT) the MMAs over the first half of the keys
// go as soon as that half is stored.  `before_first` runs after the first
// wait, ahead of the first MMA.  Returns false when a wait timed out.
template <int D, int DT, typename F>
__device__ __forceinline__ bool issue_pv_handover(uint32_t p_half_bar, uint32_t p_full_bar, uint32_t parity,
                                                  uint64_t lim, uint32_t o_tmem, uint32_t p_tmem,
                                                  uint32_t v_desc, uint32_t hi, bool accumulate,
                                                  F before_first) {
  using C = Cfg<D, DT>;
  if constexpr (C::PSPLIT) {
    if (!mbar_wait(p_half_bar, parity, lim) || !before_first()) return false;
    tc_fence_after();
    issue_pv<D, DT, 0>(o_tmem, p_tmem, v_desc, hi, accumulate);
    if (!mbar_wait(p_full_bar, parity, lim)) return false;
    tc_fence_after();
    issue_pv<D, DT, 1>(o_tmem, p_tmem, v_desc, hi, true);
  } else {
    if (!mbar_wait(p_full_bar, parity, lim) || !before_first()) return false;
    tc_fence_after();
    issue_pv<D, DT>(o_tmem, p_tmem, v_desc, hi, accumulate);
  }
  return true;
}

// The MMA thread runs alone on its warp and competes for issue slots with
// the softmax warps of its sub-partition, so every instruction between two
// MMA groups delays the tensor pipe: per key block the steady state below
// issues its 32 MMAs with nothing but the four waits, four commits and the
// ring advance between them; every decision is taken once per unit.
template <int D, int DT, bool SPLIT, int MASK>
__device__ void mma_role(SharedHeader* sh, uint8_t* tiles, uint32_t tbase, const FwdParams& p) {
  using C = Cfg<D, DT, MASK>;
  constexpr uint32_t SLOT_DESC = C::TILE_BYTES >> 4;   // descriptor start-address step per ring slot
  const uint32_t ring = smem_u32(tiles + 2 * C::TILE_BYTES);
  const uint32_t q_desc0 = sdesc_sw128_lo(smem_u32(tiles), 16);
  const uint32_t k_desc0 = sdesc_sw128_lo(ring, 16);
  const uint32_t v_desc0 = sdesc_sw128_lo(ring, C::CHUNK_BYTES);
  const uint32_t kv_full0 = smem_u32(&sh->kv_full[0]);
  const uint32_t kv_empty0 = smem_u32(&sh->kv_empty[0]);
  const uint32_t s_full0 = smem_u32(&sh->s_full[0]), p_full0 = smem_u32(&sh->p_full[0]);
  const uint32_t p_half0 = smem_u32(&sh->p_half[0]);
  const uint32_t q_empty0 = smem_u32(&sh->q_empty[0]);
  const uint64_t lim = p.wait_limit_ns;
  uint32_t q_uses = 0;
  uint32_t p_waits[2] = {0, 0};
  uint32_t o_units[2] = {0, 0};
  uint32_t kslot = 0, kpar = 0;   // ring position of K_j (loads alternate K_j, V_j)
  uint32_t vslot = 0, vpar = 0;   // ring position of V_{j-1}
  bool ok = true;
  FA_TRACE_DECL;

  for (int k = 0; ok; ++k) {
    const uint32_t qs = k & 3u, qr = static_cast<uint32_t>(k) >> 2;
    if (!mbar_wait(smem_u32(&sh->uq_full[qs]), qr & 1u, lim)) {
      record_error(sh, p, ST_TIMEOUT_MMA); ok = false; break;
    }
    const int u = *reinterpret_cast<volatile int*>(&sh->uq[qs]);
    const int us = SPLIT ? *reinterpret_cast<volatile int*>(&sh->uq_split[qs]) : 0;
    mbar_arrive(smem_u32(&sh->uq_empty[qs]));
    if (u < 0) break;
    const Unit w = get_unit<SPLIT>(u, us, p);
    if (w.jhi < 0) continue;
    if (aborted(sh)) { ok = false; break; }
    if (!mbar_wait(smem_u32(&sh->q_full[0]), q_uses & 1u, lim) ||
        !mbar_wait(smem_u32(&sh->q_full[1]), q_uses & 1u, lim)) {
      record_error(sh, p, ST_TIMEOUT_MMA); ok = false; break;
    }
    ++q_uses;
    // a tile without key blocks here does not read its Q tile (it has landed)
#pragma unroll
    for (int t = 0; t < 2; ++t)
      if (!w.valid[t]) mbar_arrive(smem_u32(&sh->q_empty[t]));
    // Steady key blocks: both tiles issue PV(j-1) and S(j), j-1 is
    // neither tile's first block (O starts from zero there, after the
    // previous unit's epilogue has read it) nor its last (O is handed over),
    // and j is neither tile's last (its S releases the tile's Q buffer).
    const bool both = w.valid[0] && w.valid[1];
    const int js = both ? max(w.lo[0], w.lo[1]) + 2 : 0x7fffffff;
    const int je = both ? min(w.hi[0], w.hi[1]) - 1 : -1;
    for (int j = w.jlo; j <= w.jhi + 1 && ok; ++j) {
      const uint32_t vfull = kv_full0 + 8u * vslot, kfull = kv_full0 + 8u * kslot;
      if (j >= js && j <= je) {
        const uint32_t v_desc = opaque(v_desc0) + vslot * SLOT_DESC;
        const uint32_t k_desc = opaque(k_desc0) + kslot * SLOT_DESC;
        const uint32_t hi = opaque(DESC_HI);
        FA_TRACE(2, 0, j);
        if (!mbar_wait(vfull, vpar, lim) ||
            !issue_pv_handover<D, DT>(p_half0, p_full0, p_waits[0] & 1u, lim, tbase + C::O_COL0,
                                      tbase + C::P_OFF, v_desc, hi, true, [] { return true; })) {
          record_error(sh, p, ST_TIMEOUT_MMA); ok = false; break;
        }
        ++p_waits[0];
        FA_TRACE(2, 1, j);
        FA_TRACE(2, 2, j);
        if (!mbar_wait(kfull, kpar, lim)) {
          record_error(sh, p, ST_TIMEOUT_MMA); ok = false; break;
        }
        FA_TRACE(2, 7, j);
        tc_fence_after();
        issue_s<D, DT>(tbase, opaque(q_desc0), k_desc, hi);
        mma_commit(s_full0);
        FA_TRACE(2, 3, j);
        if (!issue_pv_handover<D, DT>(p_half0 + 8u, p_full0 + 8u, p_waits[1] & 1u, lim, tbase + C::O_COL0 + D,
                                      tbase + 128 + C::P_OFF, v_desc, hi, true, [] { return true; })) {
          record_error(sh, p, ST_TIMEOUT_MMA); ok = false; break;
        }
        ++p_waits[1];
        FA_TRACE(2, 4, j);
        mma_commit(kv_empty0 + 8u * vslot);   // last reader of V_{j-1}
        FA_TRACE(2, 5, j);
        issue_s<D, DT>(tbase + 128, opaque(q_desc0) + SLOT_DESC, k_desc, hi);
        mma_commit(s_full0 + 8u);
        mma_commit(kv_empty0 + 8u * kslot);   // last reader of K_j
        FA_TRACE(2, 6, j);
      } else {
        // General block: either tile may skip PV(j-1) or S(j) (ragged or
        // windowed ranges, the first and last blocks of a unit).  Each
        // operand is waited for right before its first MMA and its ring slot
        // released right after its last one.
        const bool has_k = j <= w.jhi;
        const bool has_v = j > w.jlo;
        bool k_ready = false, v_ready = false, k_done = !has_k, v_done = !has_v;
        const int jp = j - 1;
        const bool pv_use[2] = {w.valid[0] && jp >= w.lo[0] && jp <= w.hi[0],
                                w.valid[1] && jp >= w.lo[1] && jp <= w.hi[1]};
        const bool s_use[2] = {w.valid[0] && j >= w.lo[0] && j <= w.hi[0],
                               w.valid[1] && j >= w.lo[1] && j <= w.hi[1]};
        const uint32_t v_desc = opaque(v_desc0) + vslot * SLOT_DESC;
        const uint32_t k_desc = opaque(k_desc0) + kslot * SLOT_DESC;
        const uint32_t hi = opaque(DESC_HI);
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          if (pv_use[t]) {
            // O_t += P_t(j-1) V_{j-1}
            if (!v_ready) {
              if (!mbar_wait(vfull, vpar, lim)) {
                record_error(sh, p, ST_TIMEOUT_MMA); ok = false; break;
              }
              v_ready = true;
            }
            // (the first PV of a unit also waits until the previous unit's
            // epilogue has read O_t out)
            const uint32_t o_empty = smem_u32(&sh->o_empty[t]), o_par = (o_units[t] & 1u) ^ 1u;
            const bool first = jp == w.lo[t];
            if (!issue_pv_handover<D, DT>(p_half0 + 8u * t, p_full0 + 8u * t, p_waits[t] & 1u, lim,
                                          tbase + C::O_COL0 + D * t, tbase + 128 * t + C::P_OFF, v_desc, hi,
                                          !first, [&] { return !first || mbar_wait(o_empty, o_par, lim); })) {
              record_error(sh, p, ST_TIMEOUT_MMA); ok = false; break;
            }
            ++p_waits[t];
            if (jp == w.hi[t]) {
              mma_commit(smem_u32(&sh->o_full[t]));
              ++o_units[t];
            }
            if (t == 1 || !pv_use[1]) {
              mma_commit(kv_empty0 + 8u * vslot);   // last reader of V_{j-1}
              v_done = true;
            }
          }
          if (s_use[t]) {
            // S_t(j) = Q_t K_j^T   (issued after PV_t(j-1), which read P_t from these columns)
            if (!k_ready) {
              if (!mbar_wait(kfull, kpar, lim)) {
                record_error(sh, p, ST_TIMEOUT_MMA); ok = false; break;
              }
              k_ready = true;
              tc_fence_after();
            }
            issue_s<D, DT>(tbase + 128 * t, opaque(q_desc0) + t * SLOT_DESC, k_desc, hi);
            mma_commit(s_full0 + 8u * t);
            if (j == w.hi[t]) mma_commit(q_empty0 + 8u * t);   // the tile's last read of its Q tile
            if (t == 1 || !s_use[1]) {
              mma_commit(kv_empty0 + 8u * kslot);   // last reader of K_j
              k_done = true;
            }
          }
        }
        if (!ok) break;
        // a loaded block nobody read (not expected): release it once it has landed
        if (!k_done) {
          if (!mbar_wait(kfull, kpar, lim)) {
            record_error(sh, p, ST_TIMEOUT_MMA); ok = false; break;
          }
          mma_commit(kv_empty0 + 8u * kslot);
        }
        if (!v_done) {
          if (!mbar_wait(vfull, vpar, lim)) {
            record_error(sh, p, ST_TIMEOUT_MMA); ok = false; break;
          }
          mma_commit(kv_empty0 + 8u * vslot);
        }
      }
      if (j <= w.jhi) {
        // V_j follows K_j, and K_{j+1} follows V_j in the ring
        vslot = kslot; vpar = kpar;
        ring_next<C::STAGES>(vslot, vpar);
        kslot = vslot; kpar = vpar;
        ring_next<C::STAGES>(kslot, kpar);
      }
    }
    if (!ok) break;
  }
  FA_TRACE(2, 15, 0);
  // all issued MMAs complete before the CTA releases TMEM
  mma_commit(smem_u32(&sh->mma_done));
  if (!mbar_wait(smem_u32(&sh->mma_done), 0, lim)) record_error(sh, p, ST_TIMEOUT_DRAIN);
}

// ------------------------------------------------------------------ dropout
// Philox4x32 with 10 rounds (Salmon, Moraes, Dror, Shaw, "Parallel Random
// Numbers: As Easy as 1, 2, 3", SC 2011): each round multiplies counter
// words 0 and 2 by two fixed odd constants and mixes the high and low
// halves of the products with words 1 and 3 and the key; the key is bumped
// by two Weyl constants between rounds.
__device__ __forceinline__ uint4 philox4x32_10(uint4 c, const PhiloxKeys& key) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const uint32_t hi0 = __umulhi(0xD2511F53u, c.x), lo0 = 0xD2511F53u * c.x;
    const uint32_t hi1 = __umulhi(0xCD9E8D57u, c.z), lo1 = 0xCD9E8D57u * c.z;
    c = make_uint4(hi1 ^ c.y ^ key.k0[r], lo1, hi0 ^ c.w ^ key.k1[r], lo0);
  }
  return c;
}

// Keep bits of 8 consecutive keys 8g .. 8g+7 of one row: bit e for key
// 8g + e, from the 16-bit halves of the four output words (low half first).
__device__ __forceinline__ uint32_t keep_bits8(uint32_t g, uint32_t row, uint32_t bh, uint32_t offset,
                                               const PhiloxKeys& key, uint32_t t) {
  const uint4 w = philox4x32_10(make_uint4(g, row, bh, offset), key);
  const uint32_t words[4] = {w.x, w.y, w.z, w.w};
  uint32_t bits = 0;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    bits |= ((words[e] & 0xffffu) >= t ? 1u : 0u) << (2 * e);
    bits |= ((words[e] >> 16) >= t ? 1u : 0u) << (2 * e + 1);
  }
  return bits;
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

// Two e4m3 values (low 16 bits) back to fp32.
__device__ __forceinline__ float2 unpack2_e4m3(uint32_t bits) {
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(bits), __NV_E4M3);
  return __half22float2(*reinterpret_cast<const __half2*>(&h));
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

// 16 fp32 values times inv -> four 16-byte stores (slice partials)
__device__ __forceinline__ void store_part_row16(float* dst, const float* o, float inv) {
#pragma unroll
  for (int i = 0; i < 4; ++i)
    reinterpret_cast<float4*>(dst)[i] =
        make_float4(o[4 * i] * inv, o[4 * i + 1] * inv, o[4 * i + 2] * inv, o[4 * i + 3] * inv);
}

// Coefficients of 2^f on f in [-1/2, 1/2], fitted by the Remez exchange on
// relative error (csrc/gen_exp2_poly.py): degree 3, max relative error
// 7.5e-5 (below the 16-bit P rounding); degree 2, 1.7e-3 (far below e4m3's);
// degree 5, 2.2e-7 (as close as ex2.approx itself, for the backward, whose
// P also enters dS in fp32).

// 2^x on the FMA pipe for a pair of finite x (unmasked blocks only).
// Range reduction for base 2 is exact: x = j + f with j = round(x) and
// f in [-1/2, 1/2]; 2^j is added into the exponent field and 2^f is the
// polynomial above.  x is clamped to -125 first so 2^j stays a normal
// number; those terms are < 2^-124.
template <int DEG>
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
  constexpr float kRound = 12582912.0f;   // 1.5 * 2^23: adding it rounds to an integer
  x.x = fmaxf(x.x, -125.0f);
  x.y = fmaxf(x.y, -125.0f);
  const float2 t = __fadd2_rn(x, make_float2(kRound, kRound));
  const float2 j = __fadd2_rn(t, make_float2(-kRound, -kRound));
  const float2 f = __ffma2_rn(j, make_float2(-1.0f, -1.0f), x);
  float2 q;
  if constexpr (DEG == 5) {
    q = __ffma2_rn(make_float2(0.0013276472454890609f, 0.0013276472454890609f), f,
                   make_float2(0.009675540961325169f, 0.009675540961325169f));
    q = __ffma2_rn(q, f, make_float2(0.05550713092088699f, 0.05550713092088699f));
    q = __ffma2_rn(q, f, make_float2(0.24022120237350464f, 0.24022120237350464f));
    q = __ffma2_rn(q, f, make_float2(0.6931469440460205f, 0.6931469440460205f));
    q = __ffma2_rn(q, f, make_float2(1.0000001192092896f, 1.0000001192092896f));
  } else if constexpr (DEG == 3) {
    q = __ffma2_rn(make_float2(0.0551716685295105f, 0.0551716685295105f), f,
                   make_float2(0.2426111251115799f, 0.2426111251115799f));
    q = __ffma2_rn(q, f, make_float2(0.6932609677314758f, 0.6932609677314758f));
    q = __ffma2_rn(q, f, make_float2(0.9999280571937561f, 0.9999280571937561f));
  } else {
    static_assert(DEG == 2, "polynomial degree");
    q = __ffma2_rn(make_float2(0.23842893540859222f, 0.23842893540859222f), f,
                   make_float2(0.7034479975700378f, 0.7034479975700378f));
    q = __ffma2_rn(q, f, make_float2(1.0004431009292603f, 1.0004431009292603f));
  }
  // t's low mantissa bits hold j; shifting by 23 moves j into the exponent field
  return make_float2(__uint_as_float(__float_as_uint(q.x) + (__float_as_uint(t.x) << 23)),
                     __uint_as_float(__float_as_uint(q.y) + (__float_as_uint(t.y) << 23)));
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Exponentiate chunks [Q0, Q0+NQ) of 16 of this thread's 64 scores of a
// row, write P (16-bit or e4m3)
// into TMEM at p_addr (16x32bx2 layout: lanes 0-15 of the access for
// threads 0-15, the same lanes half a row of P further for threads 16-31)
// and return their fp32 sum twice: exact, and over the values P*V uses
// (different only for e4m3, whose 3-bit mantissa would otherwise bias O).
// With EMULATE (blocks without masked keys), pairs i >= EMU_FROM of every 8
// take exp2_poly2 on the FMA pipe instead of MUFU.
template <int DT, bool EMULATE, int Q0, int NQ, int EMU_FROM = 8, int EMU_DEG = 3, bool DROP = false>
__device__ __forceinline__ float2 exp_half(const float* s, float cc, float neg_mref, uint32_t p_addr,
                                           const uint32_t* keep = nullptr) {
  const float2 cc2 = make_float2(cc, cc);
  const float2 nm2 = make_float2(neg_mref, neg_mref);
  float2 acc[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
  float2 accq = make_float2(0.f, 0.f);   // e4m3 only: sum of the rounded values
#pragma unroll
  for (int q = Q0; q < Q0 + NQ; ++q) {
    uint32_t pw[8];
    float2 prev = make_float2(0.f, 0.f);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int c = q * 16 + 2 * i;
      const float2 x = __ffma2_rn(make_float2(s[c], s[c + 1]), cc2, nm2);
      float2 e;
      if (EMULATE && i >= EMU_FROM) {
        e = exp2_poly2<EMU_DEG>(x);
      } else {
        e = make_float2(ex2_approx(x.x), ex2_approx(x.y));
      }
      acc[i & 1] = __fadd2_rn(acc[i & 1], e);
      if constexpr (DROP) {
        // dropped keys add nothing to P V (the row sum keeps them)
        const uint32_t kb = keep[c / 32] >> (c % 32);
        e.x = (kb & 1u) ? e.x : 0.f;
        e.y = (kb & 2u) ? e.y : 0.f;
      }
      if constexpr (DT == DT_E4M3) {
        if (i & 1) {
          pw[i / 2] = pack4_e4m3(prev.x, prev.y, e.x, e.y);
          accq = __fadd2_rn(accq, __fadd2_rn(unpack2_e4m3(pw[i / 2] & 0xffffu), unpack2_e4m3(pw[i / 2] >> 16)));
        } else {
          prev = e;
        }
      } else {
        pw[i] = pack2<DT>(e.x, e.y);
      }
    }
    if constexpr (DT == DT_E4M3) {
      tmem_st_16x32bx2_x4<16>(p_addr + q * 4, pw);   // 16 e4m3 values = 4 columns
    } else {
      tmem_st_16x32bx2_x8<32>(p_addr + q * 8, pw);
    }
  }
  const float2 a = __fadd2_rn(acc[0], acc[1]);
  const float exact = a.x + a.y;
  // (exact sum for the log-sum-exp, sum of the values P*V uses for O)
  return make_float2(exact, DT == DT_E4M3 ? accq.x + accq.y : exact);
}

// Softmax role.  Eight warps per Q tile t; warp (quad, sub) owns the 16
// rows 32*quad + 16*sub .. +15 (TMEM lanes), and inside the warp lanes 0-15
// take score columns [0, 64) of those rows, lanes 16-31 columns [64, 128)
// (the tcgen05 16x32bx2 access shape), so the two halves of a row meet with
// one shuffle and apply identical references and rescale factors.
template <int D, int DT, bool SPLIT, int MASK>
__device__ void softmax_role(SharedHeader* sh, const uint8_t* tiles, uint32_t tbase, const int t, const int sub,
                             const FwdParams& p) {
  using C = Cfg<D, DT, MASK>;
  uint32_t m_cnt = 0;   // mask tiles of this Q tile consumed (the producer's sequence)
  constexpr int HALF_N = BLOCK_N / 2;
  constexpr int HALF_D = D / 2;
  const int quad = (threadIdx.x / 32) & 3;
  const int half = static_cast<int>(lane_id()) >> 4;
  const int r = quad * 32 + sub * 16 + (static_cast<int>(lane_id()) & 15);   // row in tile
  const uint32_t lane_off = static_cast<uint32_t>(quad * 32 + sub * 16) << 16;
  const uint32_t s_addr = tbase + lane_off + t * 128;
  const uint32_t p_addr = tbase + lane_off + t * 128 + C::P_OFF;
  const uint32_t o_addr = tbase + lane_off + C::O_COL0 + t * D;
  const float cc = p.score_scale;
  FA_TRACE_DECL;
  uint32_t s_waits = 0, units = 0;
  bool ok = true;
  constexpr int OUT_ES = 2;

  for (int k = 0; ok; ++k) {
    const uint32_t qs = k & 3u, qr = static_cast<uint32_t>(k) >> 2;
    bool have = mbar_wait(smem_u32(&sh->uq_full[qs]), qr & 1u, p.wait_limit_ns);
    have = __all_sync(0xffffffffu, have);
    if (!have) { record_error(sh, p, ST_TIMEOUT_SOFTMAX); ok = false; break; }
    const int u = *reinterpret_cast<volatile int*>(&sh->uq[qs]);
    const int us = SPLIT ? *reinterpret_cast<volatile int*>(&sh->uq_split[qs]) : 0;
    __syncwarp();
    if (lane_id() == 0) mbar_arrive(smem_u32(&sh->uq_empty[qs]));
    FA_TRACE(t, 8, 0);
    if (u < 0) break;
    const Tile w = get_tile<SPLIT>(u, us, t, p);
    if (!w.rows) continue;
    const int row = w.qs + r;
    const bool row_ok = row < w.nq;
    // this row's O and LSE elements (in the output, or in this key slice's
    // partials, which hold part_rows() more rows per slice), from a tile
    // recomputed where they are used, so nothing extra stays live through
    // the block loop
    auto o_elem = [&](const Tile& x) {
      return ((x.orow0 + row) * p.H + x.h) * (int64_t)D + half * HALF_D;
    };
    auto l_elem = [&](const Tile& x) { return x.lse0 + row; };
    auto part_rows = [&]() { return static_cast<int64_t>(w.split) * p.B * p.Nq * p.H; };
    if (!w.valid) {
      // no visible key for any row of this tile (in this slice)
      if (row_ok) {
        float z[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) z[i] = 0.f;
        if constexpr (SPLIT) {
#pragma unroll
          for (int c = 0; c < HALF_D; c += 16) store_part_row16(p.o_part + part_rows() * D + o_elem(w) + c, z, 0.f);
          if (half == 0) p.lse_part[part_rows() + l_elem(w)] = -INFINITY;
        } else {
          uint8_t* out_row = reinterpret_cast<uint8_t*>(p.out) + o_elem(w) * OUT_ES;
#pragma unroll
          for (int c = 0; c < HALF_D; c += 16) store_out_row16<DT>(out_row + c * OUT_ES, z, 0.f);
          if (p.lse && half == 0) p.lse[l_elem(w)] = -INFINITY;
        }
      }
      continue;
    }
    if (aborted(sh)) { ok = false; break; }
    float m_used = -INFINITY;   // reference max (log2 units) that P and l are taken against
    float l = 0.f;              // this thread's share of the row sum (exact)
    float lq = 0.f;             // ... of the stored P values (differs for e4m3)
    constexpr bool ATTN_MASK = C::TMA_MASK;
    constexpr bool DROP = MASK == MASK_DROPOUT;
    for (int j = w.lo; j <= w.hi; ++j) {
      // boundary blocks (causal diagonal or right window edge, left window
      // edge, key tail), decided before S arrives
      const int k0 = j * BLOCK_N;
      const bool need_mask = (k0 + BLOCK_N > w.nk) ||
                             (p.window_right >= 0 && k0 + BLOCK_N - 1 > w.qs + p.window_right) ||
                             (p.window_left >= 0 && k0 < w.qs + BLOCK_M - 1 - p.window_left);
      // dropout keep bits of this thread's keys (bit c: key k0 + 64 * half + c),
      // generated while S is computed
      uint32_t keep[2] = {0u, 0u};
      if constexpr (DROP) {
        const uint32_t g0 = static_cast<uint32_t>(k0 + half * HALF_N) / 8u;
        const uint32_t bh = static_cast<uint32_t>(w.b * p.H + w.h);
#pragma unroll
        for (int g = 0; g < HALF_N / 8; ++g)
          keep[g / 4] |= keep_bits8(g0 + g, static_cast<uint32_t>(row), bh, p.drop_offset, p.drop_keys,
                                    p.drop_threshold)
                         << (8 * (g % 4));
      }
      bool got = mbar_wait(smem_u32(&sh->s_full[t]), s_waits & 1u, p.wait_limit_ns);
      got = __all_sync(0xffffffffu, got);
      if (!got) { record_error(sh, p, ST_TIMEOUT_SOFTMAX); ok = false; break; }
      ++s_waits;
      tc_fence_after();
      FA_TRACE(t, 1, j);
      float s[HALF_N];
      tmem_ld_16x32bx2_x32<64>(s_addr + 0, reinterpret_cast<uint32_t*>(s + 0));
      tmem_ld_16x32bx2_x32<64>(s_addr + 32, reinterpret_cast<uint32_t*>(s + 32));
      tmem_wait_ld();
      FA_TRACE(t, 2, j);
      // this block's mask values for the thread's 64 keys, from the tile's
      // slot (staged by the producer's TMA, 128-byte swizzled: 16-byte unit
      // u of row r at u ^ (r mod 8)), applied one 16-byte unit at a time;
      // the slot is released once read
      if constexpr (ATTN_MASK) {
        const uint32_t ms = C::M_SLOTS == 1 ? 0u : (m_cnt & 1u);
        const uint32_t mpar = (C::M_SLOTS == 1 ? m_cnt : (m_cnt >> 1)) & 1u;
        ++m_cnt;
        bool got_m = mbar_wait(smem_u32(&sh->m_full[t][ms]), mpar, p.wait_limit_ns);
        got_m = __all_sync(0xffffffffu, got_m);
        if (!got_m) { record_error(sh, p, ST_TIMEOUT_SOFTMAX); ok = false; break; }
        // boolean: the row's 128 bytes, keys 64 * half on in units 4 * half ..;
        // additive: column chunk `half` (64 keys of 2 bytes), units 0-7
        const uint8_t* mrow = tiles + C::OFF_MASK + (t * C::M_SLOTS + ms) * C::M_TILE +
                              (C::MES == 2 ? half * C::CHUNK_BYTES : 0) + r * 128;
        constexpr int KEYS_PER_UNIT = 16 / C::MES;
#pragma unroll
        for (int c0 = 0; c0 < HALF_N; c0 += KEYS_PER_UNIT) {
          const int u = (C::MES == 2 ? 0 : 4 * half) + c0 / KEYS_PER_UNIT;
          const uint4 v4 = *reinterpret_cast<const uint4*>(mrow + ((u ^ (r & 7)) << 4));
          const uint32_t wd[4] = {v4.x, v4.y, v4.z, v4.w};
          if constexpr (MASK == MASK_BOOL) {
            // byte i: key k0 + 64 * half + c0 + i; 0 = masked out
#pragma unroll
            for (int i = 0; i < 16; ++i)
              if (((wd[i / 4] >> (8 * (i % 4))) & 0xffu) == 0u) s[c0 + i] = -INFINITY;
          } else {
            // the additive mask goes into the raw score: s + m / (scale * descales)
#pragma unroll
            for (int i = 0; i < 8; i += 2) {
              float2 m2;
              if constexpr (DT == DT_FP16) {
                m2 = __half22float2(*reinterpret_cast<const __half2*>(&wd[i / 2]));
              } else {
                m2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wd[i / 2]));
              }
              s[c0 + i] = fmaf(m2.x, p.mask_scale, s[c0 + i]);
              s[c0 + i + 1] = fmaf(m2.y, p.mask_scale, s[c0 + i + 1]);
            }
          }
        }
        mbar_arrive(smem_u32(&sh->m_empty[t][ms]));
      }
      if (need_mask) {
        const int kh = k0 + half * HALF_N;
        const int hi_c = min(w.nk - kh, p.window_right >= 0 ? row + p.window_right - kh + 1 : HALF_N);
        const int lo_c = p.window_left >= 0 ? row - p.window_left - kh : 0;
#pragma unroll
        for (int c = 0; c < HALF_N; ++c)
          if (c < lo_c || c >= hi_c) s[c] = -INFINITY;
      }
      // half-row max (8 chains of 3-input max), then the other half's lane
      float mx8[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) mx8[q] = fmaxf(s[q], s[8 + q]);
#pragma unroll
      for (int c = 16; c < HALF_N; c += 16)
#pragma unroll
        for (int q = 0; q < 8; ++q) mx8[q] = fmax3(mx8[q], s[c + q], s[c + 8 + q]);
      const float mx_half = fmaxf(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(fmax3(mx8[3], mx8[4], mx8[5]), mx8[6], mx8[7]));
      const float mx = fmaxf(mx_half, __shfl_xor_sync(0xffffffffu, mx_half, 16));
      const float m_blk = mx * cc;   // -inf stays -inf (cc > 0)
      const float m_cand = fmaxf(m_used, m_blk);
      const bool need = m_cand > m_used + C::RESCALE_THRESHOLD;
      const bool warp_rescale = __any_sync(0xffffffffu, need);
      // The new reference is a select, so the exponentials start right
      // away; alpha, which rescales O and l from the old reference to the
      // new one (one MUFU op, rarely needed), is taken after them.
      const float m_old = m_used;
      m_used = warp_rescale ? m_cand : m_used;
      const float mref = (m_used == -INFINITY) ? 0.f : (m_used - C::PSHIFT);
      FA_TRACE(t, 3, j);
      // chunks of 16 scores exponentiated before the first hand-over: with
      // the split hand-over, P over keys k with k mod 64 < 32 goes first
      constexpr int NQ0 = C::PSPLIT ? 2 : 4;
      float2 lsum = need_mask ? exp_half<DT, false, 0, NQ0, 8, 3, DROP>(s, cc, -mref, p_addr, keep)
                              : exp_half<DT, true, 0, NQ0, C::EMU_FROM, C::EMU_DEG, DROP>(s, cc, -mref, p_addr, keep);
      float alpha = 1.f;
      if (warp_rescale) alpha = (m_cand == -INFINITY) ? 1.f : ex2_approx(m_old - m_cand);
      // O rescale of this thread's half row (only when some row of this warp
      // raised its reference); PV_t(j-1) has completed: S_t(j) was issued
      // after it and has landed.
      if (warp_rescale && j > w.lo) {
        const float2 a2 = make_float2(alpha, alpha);
#pragma unroll
        for (int c = 0; c < HALF_D; c += 16) {
          uint32_t o[16];
          tmem_ld_16x32bx2_x16<HALF_D>(o_addr + c, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; i += 2) {
            const float2 v = __fmul2_rn(make_float2(__uint_as_float(o[i]), __uint_as_float(o[i + 1])), a2);
            o[i] = __float_as_uint(v.x);
            o[i + 1] = __float_as_uint(v.y);
          }
          tmem_st_16x32bx2_x16<HALF_D>(o_addr + c, o);
        }
      }
      if constexpr (C::PSPLIT) {
        // the first PV MMAs run while the rest of P is exponentiated; O was
        // rescaled (above) before this first hand-over
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(smem_u32(&sh->p_half[t]));
        FA_TRACE(t, 12, j);
        const float2 ls2 = need_mask ? exp_half<DT, false, 2, 2, 8, 3, DROP>(s, cc, -mref, p_addr, keep)
                                     : exp_half<DT, true, 2, 2, C::EMU_FROM, C::EMU_DEG, DROP>(s, cc, -mref, p_addr, keep);
        lsum = make_float2(lsum.x + ls2.x, lsum.y + ls2.y);
      }
      FA_TRACE(t, 4, j);
      l = fmaf(l, alpha, lsum.x);
      lq = fmaf(lq, alpha, lsum.y);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(smem_u32(&sh->p_full[t]));
      FA_TRACE(t, 5, j);
    }
    if (!ok) break;
    // epilogue: O / l, LSE; l is the sum of both half rows
    const float l_row = l + __shfl_xor_sync(0xffffffffu, l, 16);
    const float lq_row = lq + __shfl_xor_sync(0xffffffffu, lq, 16);
    bool got = mbar_wait(smem_u32(&sh->o_full[t]), units & 1u, p.wait_limit_ns);
    got = __all_sync(0xffffffffu, got);
    if (!got) { record_error(sh, p, ST_TIMEOUT_SOFTMAX); ok = false; break; }
    ++units;
    FA_TRACE(t, 6, 0);
    tc_fence_after();
    const float inv = (lq_row > 0.f ? 1.f / lq_row : 0.f) * p.out_scale;
    // the thread's whole half row of O in one round trip (its scores are
    // dead by now, so the registers are free), then O_t is released
    uint32_t o[HALF_D];
#pragma unroll
    for (int c = 0; c < HALF_D; c += 32) tmem_ld_16x32bx2_x32<HALF_D>(o_addr + c, o + c);
    tmem_wait_ld();
    tc_fence_before();
    mbar_arrive(smem_u32(&sh->o_empty[t]));
    const Tile we = get_tile<SPLIT>(static_cast<int>(opaque(static_cast<uint32_t>(u))), us, t, p);
    if (row_ok) {
      if constexpr (SPLIT) {
        float* part_row = p.o_part + part_rows() * D + o_elem(we);
#pragma unroll
        for (int c = 0; c < HALF_D; c += 16) store_part_row16(part_row + c, reinterpret_cast<float*>(o + c), inv);
      } else {
        uint8_t* out_row = reinterpret_cast<uint8_t*>(p.out) + o_elem(we) * OUT_ES;
#pragma unroll
        for (int c = 0; c < HALF_D; c += 16)
          store_out_row16<DT>(out_row + c * OUT_ES, reinterpret_cast<float*>(o + c), inv);
      }
    }
    if (row_ok && half == 0) {
      // natural log of sum_j exp(scale * s_j) = (m_used + log2(l) - PSHIFT) * ln 2
      const float lse_v = l_row > 0.f ? (m_used + __log2f(l_row) - C::PSHIFT) * 0.69314718055994531f : -INFINITY;
      if constexpr (SPLIT) p.lse_part[part_rows() + l_elem(we)] = lse_v;
      else if (p.lse) p.lse[l_elem(we)] = lse_v;
    }
    FA_TRACE(t, 7, 0);
  }
  FA_TRACE(t, 15, 0);
}

// ------------------------------------------------------------------ kernel
// Called once per CTA by thread 0 when the CTA claims no more units: the
// last CTA of the launch to get here zeroes the scheduler scratch for the
// next launch (every CTA gets here: all waits are bounded).
__device__ __forceinline__ void cta_finished(const FwdParams& p) {
  __threadfence();
  if (atomicAdd(p.sched + 1, 1u) == gridDim.x - 1) {
    atomicExch(p.sched, 0u);
    atomicExch(p.sched + 1, 0u);
    __threadfence();
  }
}

template <int D, int DT, bool SPLIT, int MASK>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_m,
                  const FwdParams p) {
  using C = Cfg<D, DT, MASK>;
  extern __shared__ __align__(1024) uint8_t smem[];
  if ((smem_u32(smem) & 1023u) != 0) {
    // 128-byte swizzled tiles need 1024-byte alignment; never expected.  The
    // CTA still counts itself finished, so the scratch is left at zero.
    griddep_wait();
    if (threadIdx.x == 0) {
      atomicOr(p.status, ST_SMEM_MISALIGNED);
      cta_finished(p);
    }
    return;
  }
  SharedHeader* sh = reinterpret_cast<SharedHeader*>(smem);
  uint8_t* tiles = smem + HEADER_BYTES + XCH_BYTES;
  const int warp = threadIdx.x / 32;

  if (threadIdx.x == 0) {
    for (int t = 0; t < 2; ++t) {
      mbar_init(smem_u32(&sh->q_full[t]), 1);
      mbar_init(smem_u32(&sh->q_empty[t]), 1);
    }
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(smem_u32(&sh->kv_full[s]), 1);
      mbar_init(smem_u32(&sh->kv_empty[s]), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(smem_u32(&sh->s_full[t]), 1);
      mbar_init(smem_u32(&sh->p_full[t]), 256);   // every thread of the tile's two softmax warpgroups
      mbar_init(smem_u32(&sh->p_half[t]), 256);
      mbar_init(smem_u32(&sh->o_full[t]), 1);
      mbar_init(smem_u32(&sh->o_empty[t]), 256);
    }
    mbar_init(smem_u32(&sh->mma_done), 1);
    for (int t = 0; t < 2; ++t)
      for (int ms = 0; ms < 2; ++ms) {
        mbar_init(smem_u32(&sh->m_full[t][ms]), 1);
        mbar_init(smem_u32(&sh->m_empty[t][ms]), 256);   // every thread of the tile's softmax warps
      }
    for (int i = 0; i < 4; ++i) {
      mbar_init(smem_u32(&sh->uq_full[i]), 1);
      mbar_init(smem_u32(&sh->uq_empty[i]), UQ_CONSUMERS);
    }
    sh->abort_flag = 0;
#ifdef FA_STATS_BUILD
    for (int i = 0; i < 64; ++i) sh->stats[i] = 0u;
#endif
    fence_mbar_init();
    tma_prefetch_map(&tm_q);
    tma_prefetch_map(&tm_k);
    tma_prefetch_map(&tm_v);
    if constexpr (C::TMA_MASK) tma_prefetch_map(&tm_m);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&sh->tmem_base), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = sh->tmem_base;
  // the prologue above touches only this CTA's shared and tensor memory; the
  // previous kernel on the stream (the scheduler counters it leaves at zero,
  // any producer of Q, K, V) is complete from here on
  griddep_wait();
  griddep_launch_dependents();

  if (warp < 4) {
    setmaxnreg_dec<REGS_LOAD_MMA>();
    if (warp == 0 && lane_id() == 0) producer_role<D, DT, SPLIT, MASK>(sh, tiles, &tm_q, &tm_k, &tm_v, &tm_m, p);
    else if (warp == 1 && lane_id() == 0) mma_role<D, DT, SPLIT, MASK>(sh, tiles, tbase, p);
  } else {
    setmaxnreg_inc<REGS_SOFTMAX>();
    // warps 4-11: tile 0, warps 12-19: tile 1; within a tile the first four
    // warps take the upper 16 rows of each lane quadrant, the next four the lower
    const int t = warp < 12 ? 0 : 1;
    const int sub = ((warp - 4) >> 2) & 1;
    softmax_role<D, DT, SPLIT, MASK>(sh, tiles, tbase, t, sub, p);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
#ifdef FA_STATS_BUILD
  if (threadIdx.x == 0)
    for (int i = 0; i < 64; ++i) atomicAdd(&g_stats[i], static_cast<unsigned long long>(sh->stats[i]));
#endif
  if (threadIdx.x == 0) cta_finished(p);
}

// Combines the key-range slices of a split forward.  One warp per output
// row (b, n, h): with slice LSEs L_s and slice outputs O_s (each normalised
// by its own row sum), LSE = log sum_s exp(L_s) and O = sum_s exp(L_s - LSE)
// O_s; a row no slice sees gets O = 0, LSE = -inf.
template <int D, int OUT_DT>
__global__ void fa_merge_kernel(const float* __restrict__ o_part, const float* __restrict__ lse_part, void* out,
                                float* lse, int splits, int B, int Nq, int H) {
  constexpr int PER_LANE = D / 32;
  const int64_t rows = static_cast<int64_t>(B) * Nq * H;
  const int lane = static_cast<int>(threadIdx.x & 31u);
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x / 32);
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x / 32) + threadIdx.x / 32; i < rows; i += warps) {
    // i enumerates (b, n, h) like O; the LSE layout is [B, H, N_q]
    const int64_t h = i % H;
    const int64_t bn = i / H;
    const int64_t n = bn % Nq;
    const int64_t b = bn / Nq;
    const int64_t l_idx = (b * H + h) * Nq + n;
    float m = -INFINITY;
    for (int s = 0; s < splits; ++s) m = fmaxf(m, lse_part[static_cast<int64_t>(s) * rows + l_idx]);
    float acc[PER_LANE];
#pragma unroll
    for (int e = 0; e < PER_LANE; ++e) acc[e] = 0.f;
    float wsum = 0.f;
    if (m != -INFINITY) {
      for (int s = 0; s < splits; ++s) {
        const float ls = lse_part[static_cast<int64_t>(s) * rows + l_idx];
        if (ls == -INFINITY) continue;
        const float wgt = expf(ls - m);
        wsum += wgt;
        const float* src = o_part + (static_cast<int64_t>(s) * rows + i) * D + lane * PER_LANE;
#pragma unroll
        for (int e = 0; e < PER_LANE; ++e) acc[e] = fmaf(wgt, src[e], acc[e]);
      }
    }
    const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
    float o[PER_LANE];
#pragma unroll
    for (int e = 0; e < PER_LANE; ++e) o[e] = acc[e] * inv;
    uint32_t packed[PER_LANE / 2];
#pragma unroll
    for (int e = 0; e < PER_LANE / 2; ++e) packed[e] = pack2<OUT_DT>(o[2 * e], o[2 * e + 1]);
    uint8_t* dst = reinterpret_cast<uint8_t*>(out) + (i * D + lane * PER_LANE) * 2;
    if constexpr (PER_LANE == 4) {
      *reinterpret_cast<uint2*>(dst) = make_uint2(packed[0], packed[1]);
    } else {
      *reinterpret_cast<uint32_t*>(dst) = packed[0];
    }
    if (lse && lane == 0) lse[l_idx] = wsum > 0.f ? m + logf(wsum) : -INFINITY;
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

// The kernel's two ways of taking 2^x, side by side: the FMA-pipe
// polynomial of the given degree (2 or 3) and MUFU's ex2.approx.ftz.
__global__ void fa_exp2_check_kernel(const float* __restrict__ x, float* __restrict__ poly,
                                     float* __restrict__ mufu, int n, int degree) {
  for (int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x); i < n; i += 2 * gridDim.x * blockDim.x) {
    const float2 v = make_float2(x[i], i + 1 < n ? x[i + 1] : 0.f);
    const float2 r = degree == 2 ? exp2_poly2<2>(v) : degree == 5 ? exp2_poly2<5>(v) : exp2_poly2<3>(v);
    poly[i] = r.x;
    mufu[i] = ex2_approx(v.x);
    if (i + 1 < n) {
      poly[i + 1] = r.y;
      mufu[i + 1] = ex2_approx(v.y);
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
