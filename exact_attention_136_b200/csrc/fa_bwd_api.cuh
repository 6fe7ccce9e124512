// Host side of the backward (included by fa_api.cu after its helpers):
// argument validation, tensor maps and the three launches of fa_bwd.
#pragma once

#include "fa_bwd_kernel.cuh"

namespace fa {
namespace {

// Workspace of the backward: D_i = rowsum(dO * O) [B, H, N_q] fp32.
size_t bwd_workspace_bytes(int B, int Nq, int H, int D) {
  (void)D;
  return static_cast<size_t>(B) * Nq * H * sizeof(float);
}

// The dK/dV kernel (one CTA per key block) and the dQ kernel (one CTA per
// query block), both after the prologue; one CTA per SM each (the dQ
// kernel's shared-memory request is raised to keep a second CTA from
// waiting on the first's tensor memory).
template <int D, int DT, bool DROP>
int launch_bwd(const void* q, const void* k, const void* v, const void* dout, const BwdParams& p,
               cudaStream_t stream, DeviceState* ds, int bit) {
  using C = BwdCfg<D>;
  constexpr int DQ_SMEM_USED = DqCfg<D>::SMEM_USED;
  constexpr int DQ_SMEM = DQ_SMEM_USED > 118 * 1024 ? DQ_SMEM_USED : 118 * 1024;
  const CUtensorMapDataType tdt = DT == DT_FP16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  CUtensorMap mq, mk, mv, mdo;
  // packed sequences: one batch of total_q / total_k rows, each sequence
  // addressed by its first row
  const int tB = p.cu_q ? 1 : p.B;
  const int tq = p.cu_q ? p.total_q : p.Nq, tk = p.cu_q ? p.total_k : p.Nk;
  if (encode_bnhd(&mq, q, tdt, 2, tB, tq, p.H, D, 64, 128) ||
      encode_bnhd(&mk, k, tdt, 2, tB, tk, p.Hkv, D, 64, 128) ||
      encode_bnhd(&mv, v, tdt, 2, tB, tk, p.Hkv, D, 64, 128) ||
      encode_bnhd(&mdo, dout, tdt, 2, tB, tq, p.H, D, 64, 128))
    return FA_ERR_CUDA;
  if (!(ds->attr_set.load(std::memory_order_acquire) & (1u << bit))) {
    if (cudaFuncSetAttribute(fa_bwd_dkdv_kernel<D, DT, DROP>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) !=
        cudaSuccess)
      return FA_ERR_CUDA;
    const int rc = set_smem_attr_once(ds, bit, fa_bwd_dq_kernel<D, DT, DROP>, DQ_SMEM);
    if (rc != FA_OK) return rc;
  }
  const int64_t grid_kv = static_cast<int64_t>(p.nkb) * p.B * p.Hkv;
  const int64_t grid_q = static_cast<int64_t>(p.nqb) * p.B * p.H;
  if (grid_kv > 0x7fffffff || grid_q > 0x7fffffff) return FA_ERR_ARG;
  fa_bwd_dkdv_kernel<D, DT, DROP><<<static_cast<int>(grid_kv), BWD_THREADS, C::SMEM, stream>>>(mq, mk, mv, mdo, p);
  if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  fa_bwd_dq_kernel<D, DT, DROP><<<static_cast<int>(grid_q), BWD_THREADS, DQ_SMEM, stream>>>(mq, mk, mv, mdo, p);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

int backward(const void* q, const void* k, const void* v, const void* out, const void* dout, const float* lse,
             void* dq, void* dk, void* dv, int B, int Nq, int Nk, int H, int Hkv, int D, float scale, int causal,
             int window_left, int dtype, void* workspace, size_t workspace_bytes, cudaStream_t stream,
             float dropout_p = 0.f, unsigned long long seed = 0, unsigned offset = 0, int window_right = -1,
             const int* cu_q = nullptr, const int* cu_k = nullptr, int total_q = 0, int total_k = 0) {
  // the tensors' rows: B x N_q / N_k, or one batch of total_q / total_k
  // packed rows (N_q, N_k then the longest sequences, validated by the
  // packed entry point)
  const int rB = cu_q ? 1 : B, rNq = cu_q ? total_q : Nq, rNk = cu_q ? total_k : Nk;
  int rc = validate(q, k, v, const_cast<void*>(out), rB, rNq, rNk, H, D, scale, causal, window_left, dtype, Hkv);
  if (rc != FA_OK) return rc;
  int R = -1;
  rc = right_bound(causal, window_right, Nq, Nk, &R);
  if (rc != FA_OK) return rc;
  if (dtype == FA_E4M3) return FA_ERR_UNSUPPORTED;
  if (!(dropout_p >= 0.f && dropout_p < 1.f)) return FA_ERR_ARG;
  const bool drop = dropout_p > 0.f;
  if ((rNq > 0 && (!dout || !lse || !dq)) || (rNk > 0 && (!dk || !dv))) return FA_ERR_ARG;
  if (!aligned16(dout) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u) != 0)
    return FA_ERR_ALIGN;
  const size_t ws = bwd_workspace_bytes(rB, rNq, H, D);
  if (ws > 0 && (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 || workspace_bytes < ws))
    return FA_ERR_ARG;
  if (rNq == 0 && rNk == 0) return FA_OK;
  DeviceState* ds = nullptr;
  rc = device_state(&ds);
  if (rc != FA_OK) return rc;
  if (rNq == 0) {
    // no query sees any key: dK = dV = 0
    const size_t kv_bytes = static_cast<size_t>(rB) * rNk * Hkv * D * 2;
    if (cudaMemsetAsync(dk, 0, kv_bytes, stream) != cudaSuccess || cudaMemsetAsync(dv, 0, kv_bytes, stream) != cudaSuccess)
      return FA_ERR_CUDA;
    return FA_OK;
  }
  float* delta = static_cast<float*>(workspace);
  const int64_t rows = static_cast<int64_t>(rB) * rNq * H;
  {
    // ([B, H, N_q], or [H, total_q] like the packed forward's LSE)
    const int64_t want = (rows * (D / 8) + 255) / 256;   // D / 8 threads per row
    const int blocks = static_cast<int>(want < 8 * 148 ? want : 8 * 148);
    if (D == 64) fa_bwd_prologue_kernel<64><<<blocks, 256, 0, stream>>>(out, dout, dtype, delta, rB, rNq, H);
    else fa_bwd_prologue_kernel<128><<<blocks, 256, 0, stream>>>(out, dout, dtype, delta, rB, rNq, H);
    if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  }
  if (rNk == 0) {
    // no key: dQ = 0
    if (cudaMemsetAsync(dq, 0, static_cast<size_t>(rows) * D * 2, stream) != cudaSuccess) return FA_ERR_CUDA;
    return FA_OK;
  }
  {
    BwdParams p{};
    p.dk = dk;
    p.dv = dv;
    p.dq = dq;
    p.lse = lse;
    p.delta = delta;
    p.B = B;
    p.Nq = Nq;
    p.Nk = Nk;
    p.H = H;
    p.Hkv = Hkv;
    p.qpk = H / Hkv;
    p.causal = causal;
    p.window_left = window_left;
    p.window_right = R;
    p.scale = scale;
    p.score_scale = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
    p.nkb = (Nk + 127) / 128;
    p.nqb = (Nq + 127) / 128;
    p.cu_q = cu_q;
    p.cu_k = cu_k;
    p.total_q = total_q;
    p.total_k = total_k;
    p.wait_limit_ns = g_wait_limit_ns;
    p.status = ds->status;
    if (drop) {
      // the forward's keep rule (fa_fwd_dropout) and 1 / (1 - p)
      p.drop_threshold = static_cast<unsigned>(std::nearbyint(static_cast<double>(dropout_p) * 65536.0));
      p.seed_lo = static_cast<unsigned>(seed & 0xffffffffull);
      p.seed_hi = static_cast<unsigned>(seed >> 32);
      p.drop_keys = philox_round_keys(p.seed_lo, p.seed_hi);
      p.drop_offset = offset;
      p.drop_scale = static_cast<float>(1.0 / (1.0 - static_cast<double>(dropout_p)));
    }
    switch ((dtype * 2 + (D == 128 ? 1 : 0)) * 2 + (drop ? 1 : 0)) {
      case (FA_FP16 * 2 + 0) * 2 + 0: rc = launch_bwd<64, DT_FP16, false>(q, k, v, dout, p, stream, ds, 20); break;
      case (FA_FP16 * 2 + 1) * 2 + 0: rc = launch_bwd<128, DT_FP16, false>(q, k, v, dout, p, stream, ds, 21); break;
      case (FA_BF16 * 2 + 0) * 2 + 0: rc = launch_bwd<64, DT_BF16, false>(q, k, v, dout, p, stream, ds, 22); break;
      case (FA_BF16 * 2 + 1) * 2 + 0: rc = launch_bwd<128, DT_BF16, false>(q, k, v, dout, p, stream, ds, 23); break;
      case (FA_FP16 * 2 + 0) * 2 + 1: rc = launch_bwd<64, DT_FP16, true>(q, k, v, dout, p, stream, ds, 28); break;
      case (FA_FP16 * 2 + 1) * 2 + 1: rc = launch_bwd<128, DT_FP16, true>(q, k, v, dout, p, stream, ds, 29); break;
      case (FA_BF16 * 2 + 0) * 2 + 1: rc = launch_bwd<64, DT_BF16, true>(q, k, v, dout, p, stream, ds, 30); break;
      case (FA_BF16 * 2 + 1) * 2 + 1: rc = launch_bwd<128, DT_BF16, true>(q, k, v, dout, p, stream, ds, 31); break;
      default: return FA_ERR_UNSUPPORTED;
    }
    if (rc != FA_OK) return rc;
  }
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

}  // namespace
}  // namespace fa
