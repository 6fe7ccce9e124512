// C ABI of the attention library (declared in include/fa.h): argument
// validation, TMA tensor-map encoding, persistent-grid sizing and launch.
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <atomic>
#include <mutex>
#include <unordered_map>
#include <vector>

#include "../../include/fa.h"
#include "fa_fwd_kernel.cuh"
#include "tmap.h"

namespace fa {

__device__ int g_status_word;

// Scratch of fa_fwd_noalloc: the work scheduler's two 32-bit counters (next
// unit, finished CTAs) live in this fixed array instead of memory from
// cudaMalloc.  256 bytes, held by every GPU that loads the library until the
// process exits; only the first two words are used, for any problem size.
constexpr int kNoAllocScratchWords = 64;
constexpr int kSchedWordsNeeded = 2;
static __device__ __align__(256) unsigned g_noalloc_scratch[kNoAllocScratchWords];

namespace {

constexpr int kMaxDevices = 64;

// Scheduler scratch: one {next unit, finished CTAs} pair of counters per
// stream.  Launches on one stream run in order, launches on different
// streams use different counters, and each launch leaves its counters at
// zero.  Pairs come from chunks of kSchedSlots allocated once each; when a
// chunk is used up the next stream gets a pair from a new chunk, so no two
// streams ever share one.  A pair is zeroed on its stream when the stream
// first gets it (cudaMalloc'd memory starts undefined).
constexpr int kSchedSlots = 256;

struct DeviceState {
  std::atomic<bool> init{false};
  int num_sms = 0;
  int* status = nullptr;                 // device address of g_status_word
  std::atomic<unsigned> attr_set{0};     // bit per kernel instantiation with its attributes set
  std::vector<unsigned*> sched_chunks;   // kSchedSlots pairs each
  std::unordered_map<cudaStream_t, unsigned*> sched_slot;
  int used_in_last_chunk = kSchedSlots;
  unsigned* noalloc_scratch = nullptr;   // device address of g_noalloc_scratch
};

DeviceState g_dev[kMaxDevices];
std::mutex g_mu;
unsigned long long g_wait_limit_ns = 2000000000ull;

int device_state(DeviceState** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FA_ERR_CUDA;
  DeviceState& s = g_dev[dev];
  if (!s.init.load(std::memory_order_acquire)) {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!s.init.load(std::memory_order_relaxed)) {
      if (cudaDeviceGetAttribute(&s.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return FA_ERR_CUDA;
      if (cudaGetSymbolAddress(reinterpret_cast<void**>(&s.status), g_status_word) != cudaSuccess)
        return FA_ERR_CUDA;
      s.init.store(true, std::memory_order_release);
    }
  }
  *out = &s;
  return FA_OK;
}

int sched_counters(DeviceState* ds, cudaStream_t stream, unsigned** out) {
  std::lock_guard<std::mutex> lock(g_mu);
  auto it = ds->sched_slot.find(stream);
  if (it != ds->sched_slot.end()) {
    *out = it->second;
    return FA_OK;
  }
  if (ds->used_in_last_chunk == kSchedSlots) {
    unsigned* chunk = nullptr;
    if (cudaMalloc(&chunk, sizeof(unsigned) * 2 * kSchedSlots) != cudaSuccess) return FA_ERR_CUDA;
    ds->sched_chunks.push_back(chunk);
    ds->used_in_last_chunk = 0;
  }
  unsigned* pair = ds->sched_chunks.back() + 2 * ds->used_in_last_chunk;
  // zeroed on the stream that will use it, ahead of its first kernel
  if (cudaMemsetAsync(pair, 0, 2 * sizeof(unsigned), stream) != cudaSuccess) return FA_ERR_CUDA;
  ++ds->used_in_last_chunk;
  ds->sched_slot[stream] = pair;
  *out = pair;
  return FA_OK;
}

// Sets the shared-memory attribute of a kernel instantiation once per device
// (concurrent first calls may both set it, which is harmless).
template <typename K>
int set_smem_attr_once(DeviceState* ds, int bit, K kernel, int smem_bytes) {
  if (ds->attr_set.load(std::memory_order_acquire) & (1u << bit)) return FA_OK;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes) != cudaSuccess)
    return FA_ERR_CUDA;
  ds->attr_set.fetch_or(1u << bit, std::memory_order_release);
  return FA_OK;
}

// Device address of the static scratch array, looked up once per device
// with that device current.  In host code the array's name is only a
// host-side stand-in; kernels must be given this address.
int noalloc_scratch(DeviceState* ds, unsigned** out) {
  std::lock_guard<std::mutex> lock(g_mu);
  if (!ds->noalloc_scratch) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr) return FA_ERR_CUDA;
    ds->noalloc_scratch = static_cast<unsigned*>(ptr);
  }
  *out = ds->noalloc_scratch;
  return FA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

template <int D, int DT, bool SPLIT, int MASK = MASK_NONE>
int launch(const void* q, const void* k, const void* v, const FwdParams& base, cudaStream_t stream,
           DeviceState* ds, int bit, unsigned* sched_override) {
  using C = Cfg<D, DT, MASK>;
  FwdParams p = base;
  const CUtensorMapDataType tdt = DT == DT_FP16   ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                  : DT == DT_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                  : CU_TENSOR_MAP_DATA_TYPE_UINT8;
  CUtensorMap mq, mk, mv;
  // packed variable-length batches: one batch of total_q rows / total_k keys
  const int mb = p.cu_q ? 1 : p.B;
  const int mnq = p.cu_q ? p.total_q : p.Nq, mnk = p.cu_q ? p.total_k : p.Nk;
  if (encode_bnhd(&mq, q, tdt, C::ES, mb, mnq, p.H, D, C::BOX_INNER, BLOCK_M) ||
      encode_bnhd(&mk, k, tdt, C::ES, mb, mnk, p.Hkv, D, C::BOX_INNER, BLOCK_N) ||
      encode_bnhd(&mv, v, tdt, C::ES, mb, mnk, p.Hkv, D, C::BOX_INNER, BLOCK_N))
    return FA_ERR_CUDA;
  // the attention mask's map (other variants get an unused copy of Q's)
  CUtensorMap mm = mq;
  if constexpr (C::TMA_MASK) {
    const CUtensorMapDataType mdt = MASK == MASK_BOOL ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_UINT16;
    if (encode_mask(&mm, p.mask, mdt, C::MES, p.B, p.H, p.Nq, p.Nk, p.mask_sb, p.mask_sh, p.mask_sq, 128 / C::MES))
      return FA_ERR_CUDA;
  }
  if (!(ds->attr_set.load(std::memory_order_acquire) & (1u << bit))) {
    // The per-role register split (setmaxnreg) redistributes the registers
    // the CTA was launched with; it is only valid for the launch count it
    // was sized for, so a build that came out with another count is refused.
    cudaFuncAttributes fa{};
    if (cudaFuncGetAttributes(&fa, fa_fwd_kernel<D, DT, SPLIT, MASK>) != cudaSuccess) return FA_ERR_CUDA;
    if (fa.numRegs != REGS_LAUNCH) return FA_ERR_UNSUPPORTED;
    const int rc = set_smem_attr_once(ds, bit, fa_fwd_kernel<D, DT, SPLIT, MASK>, C::SMEM_BYTES);
    if (rc != FA_OK) return rc;
  }
  const int grid = p.num_units < ds->num_sms ? p.num_units : ds->num_sms;
  if (sched_override) {
    p.sched = sched_override;
  } else {
    int rc = sched_counters(ds, stream, &p.sched);
    if (rc != FA_OK) return rc;
  }
  // programmatic stream serialization: the kernel's prologue (barriers,
  // tensor memory, descriptor prefetch) may overlap the previous kernel on the
  // stream; it waits for that kernel before any global-memory access
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(NUM_THREADS);
  cfg.dynamicSmemBytes = C::SMEM_BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, fa_fwd_kernel<D, DT, SPLIT, MASK>, mq, mk, mv, mm, p) != cudaSuccess)
    return FA_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

int validate(const void* q, const void* k, const void* v, void* out, int B, int Nq, int Nk, int H,
             int D, float scale, int causal, int window_left, int dtype, int Hkv) {
  if (B < 1 || H < 1 || Nq < 0 || Nk < 0) return FA_ERR_ARG;
  if (Hkv < 1 || H % Hkv != 0) return FA_ERR_ARG;
  // q / out may be NULL only when there are no queries, k / v only when there are no keys
  if ((Nq > 0 && (!q || !out)) || (Nk > 0 && (!k || !v))) return FA_ERR_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return FA_ERR_ARG;
  if (causal != 0 && causal != 1) return FA_ERR_ARG;
  if (window_left < -1) return FA_ERR_ARG;
  if (dtype != FA_FP16 && dtype != FA_BF16 && dtype != FA_E4M3) return FA_ERR_ARG;
  if (D != 64 && D != 128) return FA_ERR_UNSUPPORTED;
  if (dtype == FA_E4M3 && D != 128) return FA_ERR_UNSUPPORTED;
  // TMA coordinates are 32-bit; keep every index well inside int range
  const int64_t rows_q = static_cast<int64_t>(B) * Nq * H;
  const int64_t rows_k = static_cast<int64_t>(B) * Nk * Hkv;
  if (rows_q > (int64_t(1) << 31) || rows_k > (int64_t(1) << 31)) return FA_ERR_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return FA_ERR_ALIGN;
  return FA_OK;
}

// The keys' upper bound j <= i + R the kernels apply (R = -1: none).  causal
// is R = 0 (a right window beside it cannot widen it); a right window that
// reaches past the last key bounds nothing.  With a bound, i + R stays in int
// range: N_q + N_k below 2^31 - 256 (else FA_ERR_ARG).
int right_bound(int causal, int window_right, int Nq, int Nk, int* R) {
  if (window_right < -1) return FA_ERR_ARG;
  *R = causal ? 0 : (window_right >= Nk ? -1 : window_right);
  if (*R > 0 && static_cast<int64_t>(Nq) + Nk >= (int64_t(1) << 31) - 256) return FA_ERR_ARG;
  return FA_OK;
}

// Sizes and pointers of a packed batch (fa_fwd_varlen, fa_bwd_varlen and the
// struct entry points), checked on the host.  The forward's work units cover
// max_q rows of every sequence; the backward's blocks also cover max_k keys.
int packed_check(const int* cu_q, const int* cu_k, int B, int max_q, int max_k, int total_q, int total_k, int H,
                 int H_kv, bool backward) {
  if (B < 1 || total_q < 0 || total_k < 0 || max_q < 0 || max_k < 0) return FA_ERR_ARG;
  if (!cu_q || !cu_k || (reinterpret_cast<uintptr_t>(cu_q) & 3u) != 0 || (reinterpret_cast<uintptr_t>(cu_k) & 3u) != 0)
    return FA_ERR_ARG;
  if ((total_q > 0 && max_q < 1) || max_q > total_q || max_k > total_k) return FA_ERR_ARG;
  if (backward && total_k > 0 && max_k < 1) return FA_ERR_ARG;
  const int64_t units = static_cast<int64_t>((max_q + 2 * BLOCK_M - 1) / (2 * BLOCK_M)) * B * H;
  const int64_t blocks_kv = static_cast<int64_t>((max_k + 127) / 128) * B * (H_kv > 0 ? H_kv : 1);
  const int64_t blocks_q = static_cast<int64_t>((max_q + 127) / 128) * B * H;
  if (units > 0x7fffffff || blocks_kv > 0x7fffffff || blocks_q > 0x7fffffff) return FA_ERR_ARG;
  return FA_OK;
}

// Workspace of a split forward: fp32 O of every slice [splits, B, N_q, H, D]
// followed by its LSE [splits, B, H, N_q].
size_t splitkv_workspace_bytes(int B, int Nq, int H, int D, int splits) {
  return static_cast<size_t>(splits) * B * Nq * H * (static_cast<size_t>(D) + 1) * sizeof(float);
}

int forward(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Nq, int Nk,
            int H, int Hkv, int D, float scale, int causal, int window_left, int dtype, float qd, float kd,
            float vd, cudaStream_t stream, unsigned* sched_override = nullptr, int splits = 1,
            void* workspace = nullptr, size_t workspace_bytes = 0, const void* mask = nullptr,
            int mask_type = 0, long long mask_sb = 0, long long mask_sh = 0, long long mask_sq = 0,
            float dropout_p = 0.f, unsigned long long seed = 0, unsigned offset = 0, const int* cu_q = nullptr,
            const int* cu_k = nullptr, int total_q = 0, int total_k = 0, int window_right = -1) {
  // (packed batches are validated by fa_fwd_varlen, with N_q and N_k the
  // longest sequences; here only their totals address the tensors)
  int rc = cu_q ? validate(q, k, v, out, 1, total_q, total_k, H, D, scale, causal, window_left, dtype, Hkv)
                : validate(q, k, v, out, B, Nq, Nk, H, D, scale, causal, window_left, dtype, Hkv);
  if (rc != FA_OK) return rc;
  int R = -1;
  rc = right_bound(causal, window_right, Nq, Nk, &R);
  if (rc != FA_OK) return rc;
  if (splits < 1) return FA_ERR_ARG;
  // dropout: 0 <= p < 1, 16-bit inputs, not combined with a mask or a split key range
  if (!(dropout_p >= 0.f && dropout_p < 1.f)) return FA_ERR_ARG;
  const bool dropout = dropout_p > 0.f;
  if (dropout && (mask_type != 0 || splits != 1)) return FA_ERR_ARG;
  if (dropout && dtype == FA_E4M3) return FA_ERR_UNSUPPORTED;
  if (mask_type != 0) {
    // byte (boolean) or 16-bit (additive) elements; every row of the mask
    // starts on a 16-byte boundary and holds N_k elements
    const long long mes = mask_type == FA_MASK_BOOL ? 1 : 2;
    if ((mask_type != FA_MASK_BOOL && mask_type != FA_MASK_ADD) || !mask || splits != 1 ||
        !aligned16(mask) || mask_sb < 0 || mask_sh < 0 || mask_sq < Nk || (mask_sb * mes) % 16 != 0 ||
        (mask_sh * mes) % 16 != 0 || (mask_sq * mes) % 16 != 0)
      return FA_ERR_ARG;
  }
  if (!(qd > 0.f) || !std::isfinite(qd) || !(kd > 0.f) || !std::isfinite(kd) || !(vd > 0.f) ||
      !std::isfinite(vd))
    return FA_ERR_ARG;
  // key-range slices: at most one per key block, none left empty
  const int nkb = (Nk + BLOCK_N - 1) / BLOCK_N;
  const int split_blocks = nkb > 0 ? (nkb + splits - 1) / splits : 1;
  const int used_splits = nkb > 0 ? (nkb + split_blocks - 1) / split_blocks : 1;
  if (used_splits > 1 && Nq > 0 &&
      (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 ||
       workspace_bytes < splitkv_workspace_bytes(B, Nq, H, D, used_splits)))
    return FA_ERR_ARG;
  if (cu_q ? total_q == 0 : Nq == 0) return FA_OK;
  DeviceState* ds = nullptr;
  rc = device_state(&ds);
  if (rc != FA_OK) return rc;
  if (cu_q ? total_k == 0 : Nk == 0) {
    // no keys anywhere: O = 0, LSE = -inf ([H, total_q] for packed batches,
    // the same layout as one batch of total_q rows)
    if (cu_q) {
      B = 1;
      Nq = total_q;
    }
    const int threads = 256;
    const int64_t rows = static_cast<int64_t>(B) * Nq * H;
    const int blocks = static_cast<int>(rows / threads + 1 < 4096 ? rows / threads + 1 : 4096);
    if (D == 64) fa_empty_kernel<64, 2><<<blocks, threads, 0, stream>>>(out, lse, B, Nq, H);
    else fa_empty_kernel<128, 2><<<blocks, threads, 0, stream>>>(out, lse, B, Nq, H);
    return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
  }
  FwdParams p{};
  p.out = out;
  p.lse = lse;
  p.B = B;
  p.Nq = Nq;
  p.Nk = Nk;
  p.H = H;
  p.Hkv = Hkv;
  p.qpk = H / Hkv;
  p.causal = causal;
  p.window_left = window_left;
  p.window_right = R;
  p.score_scale = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634 *
                                     static_cast<double>(qd) * static_cast<double>(kd));
  p.out_scale = vd;
  p.pairs = (Nq + 2 * BLOCK_M - 1) / (2 * BLOCK_M);
  p.split_blocks = split_blocks;
  p.splits = used_splits;
  if (p.splits > 1) {
    p.o_part = static_cast<float*>(workspace);
    p.lse_part = p.o_part + static_cast<size_t>(p.splits) * B * Nq * H * D;
  }
  const int64_t units = static_cast<int64_t>(p.pairs) * B * H * p.splits;
  if (units > 0x7fffffff) return FA_ERR_ARG;
  p.num_units = static_cast<int>(units);
  // scheduling groups: causal work runs longest-first across a group of
  // (batch, head) pairs; the group is sized so its K and V (bytes per head:
  // 2 * N_k * D * element size) take at most ~48 MB of the 126 MB L2 and it
  // still spans about two waves of units
  if (causal) {
    // (query heads of a group share one K/V head: count each head's share)
    const double kv_head = 2.0 * Nk * D * static_cast<double>(dtype == FA_E4M3 ? 1 : 2) / p.qpk;
    int g = static_cast<int>(48.0e6 / kv_head);
    const int want = (2 * ds->num_sms + p.pairs - 1) / p.pairs;
    g = g < want ? g : want;
    g = g < 1 ? 1 : g;
    p.group = g < B * H ? g : B * H;
  } else {
    p.group = 1;
  }
  p.wait_limit_ns = g_wait_limit_ns;
  p.status = ds->status;
  p.cu_q = cu_q;
  p.cu_k = cu_k;
  p.total_q = total_q;
  p.total_k = total_k;
  p.mask = mask;
  p.mask_sb = mask_sb;
  p.mask_sh = mask_sh;
  p.mask_sq = mask_sq;
  p.mask_scale = static_cast<float>(1.0 / (static_cast<double>(scale) * qd * kd));
  if (dropout) {
    // keep key j when its 16-bit random value is >= round(p * 65536) (ties
    // to even); kept probabilities are scaled by 1 / (1 - p)
    p.drop_threshold = static_cast<unsigned>(std::nearbyint(static_cast<double>(dropout_p) * 65536.0));
    p.seed_lo = static_cast<unsigned>(seed & 0xffffffffull);
    p.seed_hi = static_cast<unsigned>(seed >> 32);
    p.drop_keys = philox_round_keys(p.seed_lo, p.seed_hi);
    p.drop_offset = offset;
    p.out_scale = static_cast<float>(static_cast<double>(vd) / (1.0 - static_cast<double>(dropout_p)));
    switch (dtype * 2 + (D == 128 ? 1 : 0)) {
      case FA_FP16 * 2 + 0: return launch<64, DT_FP16, false, MASK_DROPOUT>(q, k, v, p, stream, ds, 24, sched_override);
      case FA_FP16 * 2 + 1: return launch<128, DT_FP16, false, MASK_DROPOUT>(q, k, v, p, stream, ds, 25, sched_override);
      case FA_BF16 * 2 + 0: return launch<64, DT_BF16, false, MASK_DROPOUT>(q, k, v, p, stream, ds, 26, sched_override);
      case FA_BF16 * 2 + 1: return launch<128, DT_BF16, false, MASK_DROPOUT>(q, k, v, p, stream, ds, 27, sched_override);
      default: return FA_ERR_UNSUPPORTED;
    }
  }
  if (mask_type != 0) {
    // masked forwards: every key block in the causal / window range is
    // computed (the mask decides inside the blocks)
    switch ((dtype * 2 + (D == 128 ? 1 : 0)) * 2 + (mask_type == FA_MASK_ADD ? 1 : 0)) {
      case (FA_FP16 * 2 + 0) * 2 + 0: return launch<64, DT_FP16, false, MASK_BOOL>(q, k, v, p, stream, ds, 10, sched_override);
      case (FA_FP16 * 2 + 1) * 2 + 0: return launch<128, DT_FP16, false, MASK_BOOL>(q, k, v, p, stream, ds, 11, sched_override);
      case (FA_BF16 * 2 + 0) * 2 + 0: return launch<64, DT_BF16, false, MASK_BOOL>(q, k, v, p, stream, ds, 12, sched_override);
      case (FA_BF16 * 2 + 1) * 2 + 0: return launch<128, DT_BF16, false, MASK_BOOL>(q, k, v, p, stream, ds, 13, sched_override);
      case (FA_E4M3 * 2 + 1) * 2 + 0: return launch<128, DT_E4M3, false, MASK_BOOL>(q, k, v, p, stream, ds, 14, sched_override);
      case (FA_FP16 * 2 + 0) * 2 + 1: return launch<64, DT_FP16, false, MASK_ADD>(q, k, v, p, stream, ds, 15, sched_override);
      case (FA_FP16 * 2 + 1) * 2 + 1: return launch<128, DT_FP16, false, MASK_ADD>(q, k, v, p, stream, ds, 16, sched_override);
      case (FA_BF16 * 2 + 0) * 2 + 1: return launch<64, DT_BF16, false, MASK_ADD>(q, k, v, p, stream, ds, 17, sched_override);
      case (FA_BF16 * 2 + 1) * 2 + 1: return launch<128, DT_BF16, false, MASK_ADD>(q, k, v, p, stream, ds, 18, sched_override);
      case (FA_E4M3 * 2 + 1) * 2 + 1: return launch<128, DT_E4M3, false, MASK_ADD>(q, k, v, p, stream, ds, 19, sched_override);
      default: return FA_ERR_UNSUPPORTED;
    }
  }
  // the split forward is its own instantiation, so the plain one carries no
  // slice bookkeeping
  const bool split = p.splits > 1;
  switch ((dtype * 2 + (D == 128 ? 1 : 0)) * 2 + (split ? 1 : 0)) {
    case (FA_FP16 * 2 + 0) * 2 + 0: rc = launch<64, DT_FP16, false>(q, k, v, p, stream, ds, 0, sched_override); break;
    case (FA_FP16 * 2 + 1) * 2 + 0: rc = launch<128, DT_FP16, false>(q, k, v, p, stream, ds, 1, sched_override); break;
    case (FA_BF16 * 2 + 0) * 2 + 0: rc = launch<64, DT_BF16, false>(q, k, v, p, stream, ds, 2, sched_override); break;
    case (FA_BF16 * 2 + 1) * 2 + 0: rc = launch<128, DT_BF16, false>(q, k, v, p, stream, ds, 3, sched_override); break;
    case (FA_E4M3 * 2 + 1) * 2 + 0: rc = launch<128, DT_E4M3, false>(q, k, v, p, stream, ds, 4, sched_override); break;
    case (FA_FP16 * 2 + 0) * 2 + 1: rc = launch<64, DT_FP16, true>(q, k, v, p, stream, ds, 5, sched_override); break;
    case (FA_FP16 * 2 + 1) * 2 + 1: rc = launch<128, DT_FP16, true>(q, k, v, p, stream, ds, 6, sched_override); break;
    case (FA_BF16 * 2 + 0) * 2 + 1: rc = launch<64, DT_BF16, true>(q, k, v, p, stream, ds, 7, sched_override); break;
    case (FA_BF16 * 2 + 1) * 2 + 1: rc = launch<128, DT_BF16, true>(q, k, v, p, stream, ds, 8, sched_override); break;
    case (FA_E4M3 * 2 + 1) * 2 + 1: rc = launch<128, DT_E4M3, true>(q, k, v, p, stream, ds, 9, sched_override); break;
    default: return FA_ERR_UNSUPPORTED;
  }
  if (rc != FA_OK || p.splits == 1) return rc;
  // combine the slices (same stream, so it runs after the forward)
  const int64_t rows = static_cast<int64_t>(B) * Nq * H;
  const int warps_per_block = 8;
  const int64_t want = (rows + warps_per_block - 1) / warps_per_block;
  const int blocks = static_cast<int>(want < 8 * 148 ? want : 8 * 148);
  const bool fp16_out = dtype == FA_FP16;
  if (D == 64) {
    if (fp16_out) fa_merge_kernel<64, DT_FP16><<<blocks, 32 * warps_per_block, 0, stream>>>(p.o_part, p.lse_part, out, lse, p.splits, B, Nq, H);
    else fa_merge_kernel<64, DT_BF16><<<blocks, 32 * warps_per_block, 0, stream>>>(p.o_part, p.lse_part, out, lse, p.splits, B, Nq, H);
  } else {
    if (fp16_out) fa_merge_kernel<128, DT_FP16><<<blocks, 32 * warps_per_block, 0, stream>>>(p.o_part, p.lse_part, out, lse, p.splits, B, Nq, H);
    else fa_merge_kernel<128, DT_BF16><<<blocks, 32 * warps_per_block, 0, stream>>>(p.o_part, p.lse_part, out, lse, p.splits, B, Nq, H);
  }
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

size_t elem_bytes(int dtype) { return dtype == FA_E4M3 ? 1 : 2; }

}  // namespace
}  // namespace fa

#include "fa_bwd_api.cuh"   // backward: validation and launches

extern "C" {

int fa_fwd(const void* q, const void* k, const void* v, void* out, float* lse, int B, int N_q, int N_k,
           int H, int D, float scale, int causal, int window_left, int dtype, fa_stream_t stream) {
  return fa::forward(q, k, v, out, lse, B, N_q, N_k, H, H, D, scale, causal, window_left, dtype, 1.f, 1.f,
                     1.f, reinterpret_cast<cudaStream_t>(stream));
}

int fa_fwd_fp8(const void* q, const void* k, const void* v, void* out, float* lse, int B, int N_q,
               int N_k, int H, int D, float scale, int causal, int window_left, float q_descale,
               float k_descale, float v_descale, fa_stream_t stream) {
  return fa::forward(q, k, v, out, lse, B, N_q, N_k, H, H, D, scale, causal, window_left, FA_E4M3,
                     q_descale, k_descale, v_descale, reinterpret_cast<cudaStream_t>(stream));
}

int fa_fwd_gqa(const void* q, const void* k, const void* v, void* out, float* lse, int B, int N_q, int N_k,
               int H, int H_kv, int D, float scale, int causal, int window_left, int dtype, float q_descale,
               float k_descale, float v_descale, fa_stream_t stream) {
  return fa::forward(q, k, v, out, lse, B, N_q, N_k, H, H_kv, D, scale, causal, window_left, dtype, q_descale,
                     k_descale, v_descale, reinterpret_cast<cudaStream_t>(stream));
}

int fa_fwd_window(const void* q, const void* k, const void* v, void* out, float* lse, int B, int N_q, int N_k,
                  int H, int H_kv, int D, float scale, int causal, int window_left, int window_right, int dtype,
                  float q_descale, float k_descale, float v_descale, fa_stream_t stream) {
  return fa::forward(q, k, v, out, lse, B, N_q, N_k, H, H_kv, D, scale, causal, window_left, dtype, q_descale,
                     k_descale, v_descale, reinterpret_cast<cudaStream_t>(stream), nullptr, 1, nullptr, 0, nullptr, 0,
                     0, 0, 0, 0.f, 0, 0, nullptr, nullptr, 0, 0, window_right);
}

size_t fa_fwd_splitkv_workspace_bytes(int B, int N_q, int N_k, int H, int D, int num_splits) {
  if (B < 1 || N_q < 0 || N_k < 0 || H < 1 || D < 1 || num_splits < 1) return 0;
  // the slices the forward will actually use
  const int nkb = (N_k + fa::BLOCK_N - 1) / fa::BLOCK_N;
  if (nkb == 0) return 0;
  const int per = (nkb + num_splits - 1) / num_splits;
  const int splits = (nkb + per - 1) / per;
  return splits > 1 ? fa::splitkv_workspace_bytes(B, N_q, H, D, splits) : 0;
}

int fa_fwd_splitkv(const void* q, const void* k, const void* v, void* out, float* lse, int B, int N_q, int N_k,
                   int H, int H_kv, int D, float scale, int causal, int window_left, int dtype, float q_descale,
                   float k_descale, float v_descale, int num_splits, void* workspace, size_t workspace_bytes,
                   fa_stream_t stream) {
  return fa::forward(q, k, v, out, lse, B, N_q, N_k, H, H_kv, D, scale, causal, window_left, dtype, q_descale,
                     k_descale, v_descale, reinterpret_cast<cudaStream_t>(stream), nullptr, num_splits, workspace,
                     workspace_bytes);
}

int fa_fwd_mask(const void* q, const void* k, const void* v, void* out, float* lse, int B, int N_q, int N_k,
                int H, int H_kv, int D, float scale, int causal, int window_left, int dtype, float q_descale,
                float k_descale, float v_descale, const void* mask, int mask_type, long long mask_stride_b,
                long long mask_stride_h, long long mask_stride_q, fa_stream_t stream) {
  if (mask_type != FA_MASK_BOOL && mask_type != FA_MASK_ADD) return FA_ERR_ARG;
  return fa::forward(q, k, v, out, lse, B, N_q, N_k, H, H_kv, D, scale, causal, window_left, dtype, q_descale,
                     k_descale, v_descale, reinterpret_cast<cudaStream_t>(stream), nullptr, 1, nullptr, 0, mask,
                     mask_type, mask_stride_b, mask_stride_h, mask_stride_q);
}

int fa_fwd_dropout(const void* q, const void* k, const void* v, void* out, float* lse, int B, int N_q, int N_k,
                   int H, int H_kv, int D, float scale, int causal, int window_left, int dtype, float dropout_p,
                   unsigned long long seed, unsigned offset, fa_stream_t stream) {
  return fa::forward(q, k, v, out, lse, B, N_q, N_k, H, H_kv, D, scale, causal, window_left, dtype, 1.f, 1.f, 1.f,
                     reinterpret_cast<cudaStream_t>(stream), nullptr, 1, nullptr, 0, nullptr, 0, 0, 0, 0, dropout_p,
                     seed, offset);
}

int fa_fwd_varlen(const void* q, const void* k, const void* v, void* out, float* lse, const int* cu_seqlens_q,
                  const int* cu_seqlens_k, int B, int max_seqlen_q, int max_seqlen_k, int total_q, int total_k, int H,
                  int H_kv, int D, float scale, int causal, int window_left, int dtype, float q_descale,
                  float k_descale, float v_descale, fa_stream_t stream) {
  const int rc = fa::packed_check(cu_seqlens_q, cu_seqlens_k, B, max_seqlen_q, max_seqlen_k, total_q, total_k, H,
                                  H_kv, false);
  if (rc != FA_OK) return rc;
  return fa::forward(q, k, v, out, lse, B, max_seqlen_q, max_seqlen_k, H, H_kv, D, scale, causal, window_left, dtype,
                     q_descale, k_descale, v_descale, reinterpret_cast<cudaStream_t>(stream), nullptr, 1, nullptr, 0,
                     nullptr, 0, 0, 0, 0, 0.f, 0, 0, cu_seqlens_q, cu_seqlens_k, total_q, total_k);
}

}  // extern "C"

namespace fa {
namespace {
// Copies in, the forward, copies out, all enqueued on `s` (fa_fwd_host and
// fa_fwd_host_async).
int host_forward(const void* q, const void* k, const void* v, void* out, float* lse, void* dq, void* dk,
                 void* dv, void* dout, float* dlse, int B, int N_q, int N_k, int H, int D, float scale,
                 int causal, int window_left, int dtype, float q_descale, float k_descale,
                 float v_descale, cudaStream_t s) {
  if (!q || !k || !v || !out) return FA_ERR_ARG;
  int rc = validate(dq, dk, dv, dout, B, N_q, N_k, H, D, scale, causal, window_left, dtype, H);
  if (rc != FA_OK) return rc;
  const size_t es = elem_bytes(dtype);
  const size_t nq = static_cast<size_t>(B) * N_q * H * D;
  const size_t nk = static_cast<size_t>(B) * N_k * H * D;
  if (cudaMemcpyAsync(dq, q, nq * es, cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaMemcpyAsync(dk, k, nk * es, cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaMemcpyAsync(dv, v, nk * es, cudaMemcpyHostToDevice, s) != cudaSuccess)
    return FA_ERR_CUDA;
  rc = forward(dq, dk, dv, dout, dlse, B, N_q, N_k, H, H, D, scale, causal, window_left, dtype, q_descale,
               k_descale, v_descale, s);
  if (rc != FA_OK) return rc;
  if (cudaMemcpyAsync(out, dout, nq * 2, cudaMemcpyDeviceToHost, s) != cudaSuccess) return FA_ERR_CUDA;
  if (lse && dlse &&
      cudaMemcpyAsync(lse, dlse, static_cast<size_t>(B) * H * N_q * sizeof(float), cudaMemcpyDeviceToHost,
                      s) != cudaSuccess)
    return FA_ERR_CUDA;
  return FA_OK;
}
}  // namespace
}  // namespace fa

extern "C" {

int fa_fwd_host(const void* q, const void* k, const void* v, void* out, float* lse, void* dq, void* dk,
                void* dv, void* dout, float* dlse, int B, int N_q, int N_k, int H, int D, float scale,
                int causal, int window_left, int dtype, float q_descale, float k_descale,
                float v_descale, fa_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int rc = fa::host_forward(q, k, v, out, lse, dq, dk, dv, dout, dlse, B, N_q, N_k, H, D, scale, causal,
                                  window_left, dtype, q_descale, k_descale, v_descale, s);
  if (rc != FA_OK) return rc;
  return cudaStreamSynchronize(s) == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

int fa_fwd_host_async(const void* q, const void* k, const void* v, void* out, float* lse, void* dq, void* dk,
                      void* dv, void* dout, float* dlse, int B, int N_q, int N_k, int H, int D, float scale,
                      int causal, int window_left, int dtype, float q_descale, float k_descale,
                      float v_descale, fa_stream_t stream) {
  return fa::host_forward(q, k, v, out, lse, dq, dk, dv, dout, dlse, B, N_q, N_k, H, D, scale, causal,
                          window_left, dtype, q_descale, k_descale, v_descale,
                          reinterpret_cast<cudaStream_t>(stream));
}

int fa_fwd_noalloc(const void* q, const void* k, const void* v, void* out, float* lse, int B, int N_q,
                   int N_k, int H, int D, float scale, int causal, int window_left, int dtype,
                   float q_descale, float k_descale, float v_descale, fa_stream_t stream) {
  int rc = fa::validate(q, k, v, out, B, N_q, N_k, H, D, scale, causal, window_left, dtype, H);
  if (rc != FA_OK) return rc;
  // the scheduler's counters index work units as 32-bit values: problems with
  // more units than that (or a scratch need above the array) are rejected
  const int64_t units = static_cast<int64_t>((N_q + 2 * fa::BLOCK_M - 1) / (2 * fa::BLOCK_M)) * B * H;
  if (fa::kSchedWordsNeeded > fa::kNoAllocScratchWords || units > 0x7fff0000LL) return FA_ERR_ARG;
  if (N_q == 0) return FA_OK;
  fa::DeviceState* ds = nullptr;
  rc = fa::device_state(&ds);
  if (rc != FA_OK) return rc;
  unsigned* scratch = nullptr;
  rc = fa::noalloc_scratch(ds, &scratch);
  if (rc != FA_OK) return rc;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // the counters must start at zero; every launch also leaves them at zero
  if (cudaMemsetAsync(scratch, 0, sizeof(unsigned) * fa::kSchedWordsNeeded, s) != cudaSuccess)
    return FA_ERR_CUDA;
  return fa::forward(q, k, v, out, lse, B, N_q, N_k, H, H, D, scale, causal, window_left, dtype, q_descale,
                     k_descale, v_descale, s, scratch);
}

size_t fa_bwd_workspace_bytes(int B, int N_q, int H, int D) {
  if (B < 1 || N_q < 0 || H < 1 || (D != 64 && D != 128)) return 0;
  return fa::bwd_workspace_bytes(B, N_q, H, D);
}

int fa_bwd(const void* q, const void* k, const void* v, const void* out, const void* dout, const float* lse,
           void* dq, void* dk, void* dv, int B, int N_q, int N_k, int H, int D, float scale, int causal,
           int window_left, int dtype, void* workspace, size_t workspace_bytes, fa_stream_t stream) {
  return fa::backward(q, k, v, out, dout, lse, dq, dk, dv, B, N_q, N_k, H, H, D, scale, causal, window_left, dtype,
                      workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

int fa_bwd_gqa(const void* q, const void* k, const void* v, const void* out, const void* dout, const float* lse,
               void* dq, void* dk, void* dv, int B, int N_q, int N_k, int H, int H_kv, int D, float scale,
               int causal, int window_left, int dtype, void* workspace, size_t workspace_bytes,
               fa_stream_t stream) {
  return fa::backward(q, k, v, out, dout, lse, dq, dk, dv, B, N_q, N_k, H, H_kv, D, scale, causal, window_left,
                      dtype, workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

int fa_bwd_window(const void* q, const void* k, const void* v, const void* out, const void* dout, const float* lse,
                  void* dq, void* dk, void* dv, int B, int N_q, int N_k, int H, int H_kv, int D, float scale,
                  int causal, int window_left, int window_right, int dtype, void* workspace, size_t workspace_bytes,
                  fa_stream_t stream) {
  return fa::backward(q, k, v, out, dout, lse, dq, dk, dv, B, N_q, N_k, H, H_kv, D, scale, causal, window_left,
                      dtype, workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream), 0.f, 0, 0,
                      window_right);
}

int fa_bwd_varlen(const void* q, const void* k, const void* v, const void* out, const void* dout, const float* lse,
                  void* dq, void* dk, void* dv, const int* cu_seqlens_q, const int* cu_seqlens_k, int B,
                  int max_seqlen_q, int max_seqlen_k, int total_q, int total_k, int H, int H_kv, int D, float scale,
                  int causal, int window_left, int dtype, void* workspace, size_t workspace_bytes,
                  fa_stream_t stream) {
  // (every row and key of a sequence lies in a launched block)
  const int rc = fa::packed_check(cu_seqlens_q, cu_seqlens_k, B, max_seqlen_q, max_seqlen_k, total_q, total_k, H,
                                  H_kv, true);
  if (rc != FA_OK) return rc;
  return fa::backward(q, k, v, out, dout, lse, dq, dk, dv, B, max_seqlen_q, max_seqlen_k, H, H_kv, D, scale, causal,
                      window_left, dtype, workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream), 0.f, 0,
                      0, -1, cu_seqlens_q, cu_seqlens_k, total_q, total_k);
}

int fa_fwd_ex(const fa_fwd_args* a, fa_stream_t stream) {
  if (!a || (a->cu_seqlens_q == nullptr) != (a->cu_seqlens_k == nullptr)) return FA_ERR_ARG;
  const bool packed = a->cu_seqlens_q != nullptr;
  if (packed) {
    const int rc = fa::packed_check(a->cu_seqlens_q, a->cu_seqlens_k, a->B, a->N_q, a->N_k, a->total_q, a->total_k,
                                    a->H, a->H_kv, false);
    if (rc != FA_OK) return rc;
  }
  return fa::forward(a->q, a->k, a->v, a->out, a->lse, a->B, a->N_q, a->N_k, a->H, a->H_kv, a->D, a->scale,
                     a->causal, a->window_left, a->dtype, a->q_descale, a->k_descale, a->v_descale,
                     reinterpret_cast<cudaStream_t>(stream), nullptr, 1, nullptr, 0, nullptr, 0, 0, 0, 0, a->dropout_p,
                     a->seed, a->offset, a->cu_seqlens_q, a->cu_seqlens_k, packed ? a->total_q : 0,
                     packed ? a->total_k : 0, a->window_right);
}

int fa_bwd_ex(const fa_bwd_args* a, fa_stream_t stream) {
  if (!a || (a->cu_seqlens_q == nullptr) != (a->cu_seqlens_k == nullptr)) return FA_ERR_ARG;
  const bool packed = a->cu_seqlens_q != nullptr;
  if (packed) {
    const int rc = fa::packed_check(a->cu_seqlens_q, a->cu_seqlens_k, a->B, a->N_q, a->N_k, a->total_q, a->total_k,
                                    a->H, a->H_kv, true);
    if (rc != FA_OK) return rc;
  }
  return fa::backward(a->q, a->k, a->v, a->out, a->dout, a->lse, a->dq, a->dk, a->dv, a->B, a->N_q, a->N_k, a->H,
                      a->H_kv, a->D, a->scale, a->causal, a->window_left, a->dtype, a->workspace, a->workspace_bytes,
                      reinterpret_cast<cudaStream_t>(stream), a->dropout_p, a->seed, a->offset, a->window_right,
                      a->cu_seqlens_q, a->cu_seqlens_k, packed ? a->total_q : 0, packed ? a->total_k : 0);
}

int fa_bwd_dropout(const void* q, const void* k, const void* v, const void* out, const void* dout,
                   const float* lse, void* dq, void* dk, void* dv, int B, int N_q, int N_k, int H, int H_kv, int D,
                   float scale, int causal, int window_left, int dtype, float dropout_p, unsigned long long seed,
                   unsigned offset, void* workspace, size_t workspace_bytes, fa_stream_t stream) {
  return fa::backward(q, k, v, out, dout, lse, dq, dk, dv, B, N_q, N_k, H, H_kv, D, scale, causal, window_left,
                      dtype, workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream), dropout_p, seed,
                      offset);
}

int fa_device_status(fa_stream_t stream, int* flags) {
  fa::DeviceState* ds = nullptr;
  int rc = fa::device_state(&ds);
  if (rc != FA_OK) return rc;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return FA_ERR_CUDA;
  int word = 0;
  if (cudaMemcpy(&word, ds->status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return FA_ERR_CUDA;
  const int zero = 0;
  if (word != 0 && cudaMemcpy(ds->status, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
    return FA_ERR_CUDA;
  if (flags) *flags = word;
  return word == 0 ? FA_OK : FA_ERR_TIMEOUT;
}

void fa_set_wait_limit_ns(unsigned long long limit_ns) {
  fa::g_wait_limit_ns = limit_ns > 0 ? limit_ns : 1ull;
}

int fa_wait_probe(unsigned long long limit_ns, fa_stream_t stream) {
  fa::DeviceState* ds = nullptr;
  int rc = fa::device_state(&ds);
  if (rc != FA_OK) return rc;
  fa::fa_wait_probe_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(limit_ns, ds->status);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

int fa_exp2_check(const float* x, float* poly, float* mufu, int n, int degree, fa_stream_t stream) {
  if (n < 0 || (degree != 2 && degree != 3 && degree != 5)) return FA_ERR_ARG;
  if (n == 0) return FA_OK;
  if (!x || !poly || !mufu) return FA_ERR_ARG;
  const int threads = 256;
  const int blocks = static_cast<int>(((n + 1) / 2 + threads - 1) / threads < 1024 ? ((n + 1) / 2 + threads - 1) / threads : 1024);
  fa::fa_exp2_check_kernel<<<blocks, threads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(x, poly, mufu, n, degree);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

const char* fa_status_string(int status) {
  switch (status) {
    case FA_OK: return "ok";
    case FA_ERR_ARG: return "invalid argument";
    case FA_ERR_UNSUPPORTED: return "unsupported head dim / dtype";
    case FA_ERR_ALIGN: return "pointer not 16-byte aligned";
    case FA_ERR_CUDA: return "CUDA runtime error";
    case FA_ERR_TIMEOUT: return "kernel wait timed out";
    default: return "unknown status";
  }
}

const char* fa_version(void) { return "0.1.0"; }

}  // extern "C"
