// api.cu -- the C ABI of include/diffattn_v2.h: argument checks, TMA descriptor encoding,
// split planning and kernel dispatch. No allocation, no state beyond a per-device cache of
// the device error word's address.

#include <cudaTypedefs.h>

#include <mutex>

#include "diffattn_v2.h"
#include "internal.h"

namespace {

// Device error word that kernels set (atomicCAS from 0) when a bounded wait expires.
__device__ int g_device_error = 0;

constexpr int kMaxDevices = 64;
std::mutex g_mu;
int* g_err_ptr[kMaxDevices] = {};
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

int status_of(cudaError_t e) { return e == cudaSuccess ? DA2_OK : DA2_ERR_CUDA; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Address of the device error word on the current device.
cudaError_t device_error_ptr(int** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_err_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_device_error);
    if (e != cudaSuccess) return e;
    g_err_ptr[dev] = static_cast<int*>(p);
  }
  *out = g_err_ptr[dev];
  return cudaSuccess;
}

cudaError_t get_encoder(PFN_cuTensorMapEncodeTiled_v12000* fn) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_encode) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
    if (e != cudaSuccess) return e;
    if (q != cudaDriverEntryPointSuccess || !p) return cudaErrorNotSupported;
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  *fn = g_encode;
  return cudaSuccess;
}

// 4-D bf16 tensor map over a [d3, d2, d1, d0] row-major array (d0 = D innermost), box
// {box0, 1, box2, 1}, 128-byte swizzle, out-of-range elements read as zero.
cudaError_t encode_bshd(CUtensorMap* map, const void* base, uint64_t D, uint64_t H, uint64_t S, uint64_t B,
                        uint32_t box0, uint32_t box2) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = nullptr;
  cudaError_t e = get_encoder(&enc);
  if (e != cudaSuccess) return e;
  const cuuint64_t dims[4] = {D, H, S, B};
  const cuuint64_t strides[3] = {D * 2, H * D * 2, S * H * D * 2};  // bytes, dims 1..3
  const cuuint32_t box[4] = {box0, 1, box2, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// Shape checks shared by prefill and decode: sizes positive, Hq even, pairs inside groups.
bool heads_ok(int Hq, int Hkv) { return Hq > 0 && Hkv > 0 && (Hq % 2) == 0 && (Hq % (2 * Hkv)) == 0; }

}  // namespace

namespace da2 {

size_t decode_workspace_bytes(int B, int T, int Hq, int Hkv, int D, int nsplit) {
  const size_t rows = static_cast<size_t>(B) * T * Hq * nsplit;
  return rows * static_cast<size_t>(D) * sizeof(float) + rows * 2 * sizeof(float) +
         (static_cast<size_t>(B) * Hkv * sizeof(int) + 15) / 16 * 16;
}

DecodeWorkspace decode_workspace_layout(void* base, int B, int T, int Hq, int D, int nsplit) {
  const size_t rows = static_cast<size_t>(B) * T * Hq * nsplit;
  DecodeWorkspace w;
  w.o = static_cast<float*>(base);
  w.ml = w.o + rows * static_cast<size_t>(D);
  w.counters = reinterpret_cast<int*>(w.ml + rows * 2);
  return w;
}

// With a sliding window only the last window (+ up to one stage before it) is read: plan the
// splits over that span when this gives no more splits than the plan for Smax, for which the
// caller's workspace is sized.
void decode_split_plan_window(int B, int Smax, int Hkv, int window, int* split_len, int* nsplit) {
  decode_split_plan(B, Smax, Hkv, split_len, nsplit);
  if (window <= 0 || window + 64 >= Smax) return;
  int L = 0, n = 0;
  decode_split_plan(B, window + 64, Hkv, &L, &n);
  if (n <= *nsplit) {
    *split_len = L;
    *nsplit = n;
  }
}

void decode_split_plan(int B, int Smax, int Hkv, int* split_len, int* nsplit) {
  // Aim for about 8 waves of 2 CTAs per SM over the (b, g) units, with splits that are a
  // multiple of the 64-token stage and between 512 and 4096 tokens long.
  const long long units = static_cast<long long>(B) * Hkv;
  const long long target_ctas = 148LL * 2 * 8;
  long long L = (static_cast<long long>(Smax) * units + target_ctas - 1) / target_ctas;
  L = ((L + 63) / 64) * 64;
  if (L < 512) L = 512;
  if (L > 4096) L = 4096;
  *split_len = static_cast<int>(L);
  *nsplit = static_cast<int>((Smax + L - 1) / L);
}

// Accessors for other translation units of the library.
cudaError_t device_error_word(int** out) { return device_error_ptr(out); }

cudaError_t encode_2d_bf16(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows, uint64_t row_bytes,
                           uint32_t box_cols, uint32_t box_rows) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = nullptr;
  cudaError_t e = get_encoder(&enc);
  if (e != cudaSuccess) return e;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t encode_out_bf16(CUtensorMap* map, void* base, uint64_t D, uint64_t H, uint64_t S, uint64_t B) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = nullptr;
  cudaError_t e = get_encoder(&enc);
  if (e != cudaSuccess) return e;
  const cuuint64_t dims[4] = {D, H, S, B};
  const cuuint64_t strides[3] = {D * 2, H * D * 2, S * H * D * 2};
  const cuuint32_t box[4] = {32, 1, 32, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t encode_bshd_bf16(CUtensorMap* map, const void* base, uint64_t D, uint64_t H, uint64_t S, uint64_t B,
                             uint32_t box0, uint32_t box2) {
  return encode_bshd(map, base, D, H, S, B, box0, box2);
}

}  // namespace da2

extern "C" {

int diffattn_v2_version(void) { return 100; }

const char* diffattn_v2_status_string(int status) {
  switch (status) {
    case DA2_OK: return "ok";
    case DA2_ERR_INVALID: return "invalid argument";
    case DA2_ERR_UNSUPPORTED: return "unsupported configuration";
    case DA2_ERR_CUDA: return "CUDA runtime error";
    case DA2_ERR_DEVICE: return "kernel reported a device-side error";
    default: return "unknown status";
  }
}

int diffattn_v2_prefill(const void* q, const void* k, const void* v, const float* lambda, void* out, int B, int S,
                        int Hq, int Hkv, int D, int causal, da2_stream_t stream) {
  if (B < 0 || S < 0 || D <= 0 || !heads_ok(Hq, Hkv)) return DA2_ERR_INVALID;
  if (causal != 0 && causal != 1) return DA2_ERR_INVALID;
  if (B == 0 || S == 0) return DA2_OK;
  if (!q || !k || !v || !lambda || !out) return DA2_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(lambda) || !aligned16(out))
    return DA2_ERR_INVALID;
  if (D != 128) return DA2_ERR_UNSUPPORTED;
  if ((S + 127) / 128 > 65535) return DA2_ERR_UNSUPPORTED;
  int* err = nullptr;
  cudaError_t e = device_error_ptr(&err);
  if (e != cudaSuccess) return DA2_ERR_CUDA;
  CUtensorMap tq, tk, tv, tkh;
  if (encode_bshd(&tq, q, D, Hq, S, B, 64, 128) != cudaSuccess) return DA2_ERR_CUDA;
  if (encode_bshd(&tk, k, D, Hkv, S, B, 64, 128) != cudaSuccess) return DA2_ERR_CUDA;
  if (encode_bshd(&tv, v, D, Hkv, S, B, 64, 128) != cudaSuccess) return DA2_ERR_CUDA;
  if (encode_bshd(&tkh, k, D, Hkv, S, B, 64, 64) != cudaSuccess) return DA2_ERR_CUDA;
  CUtensorMap to;
  if (da2::encode_out_bf16(&to, out, D, Hq / 2, S, B) != cudaSuccess) return DA2_ERR_CUDA;
  e = da2::launch_prefill(tq, tk, tv, &tkh, to, lambda, static_cast<__nv_bfloat16*>(out), err, B, S, Hq, Hkv, causal, 0,
                          nullptr, reinterpret_cast<cudaStream_t>(stream));
  return status_of(e);
}

int diffattn_v2_prefill_window(const void* q, const void* k, const void* v, const float* lambda, void* out, int B,
                               int S, int Hq, int Hkv, int D, int window, da2_stream_t stream) {
  if (B < 0 || S < 0 || D <= 0 || !heads_ok(Hq, Hkv) || window < 1) return DA2_ERR_INVALID;
  if (B == 0 || S == 0) return DA2_OK;
  if (!q || !k || !v || !lambda || !out) return DA2_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(lambda) || !aligned16(out))
    return DA2_ERR_INVALID;
  if (D != 128) return DA2_ERR_UNSUPPORTED;
  if ((S + 127) / 128 > 65535) return DA2_ERR_UNSUPPORTED;
  int* err = nullptr;
  cudaError_t e = device_error_ptr(&err);
  if (e != cudaSuccess) return DA2_ERR_CUDA;
  CUtensorMap tq, tk, tv, tkh;
  if (encode_bshd(&tq, q, D, Hq, S, B, 64, 128) != cudaSuccess) return DA2_ERR_CUDA;
  if (encode_bshd(&tk, k, D, Hkv, S, B, 64, 128) != cudaSuccess) return DA2_ERR_CUDA;
  if (encode_bshd(&tv, v, D, Hkv, S, B, 64, 128) != cudaSuccess) return DA2_ERR_CUDA;
  if (encode_bshd(&tkh, k, D, Hkv, S, B, 64, 64) != cudaSuccess) return DA2_ERR_CUDA;
  CUtensorMap to;
  if (da2::encode_out_bf16(&to, out, D, Hq / 2, S, B) != cudaSuccess) return DA2_ERR_CUDA;
  // a window of S or more keys is the plain causal mask
  e = da2::launch_prefill(tq, tk, tv, &tkh, to, lambda, static_cast<__nv_bfloat16*>(out), err, B, S, Hq, Hkv, 1,
                          window >= S ? 0 : window, nullptr, reinterpret_cast<cudaStream_t>(stream));
  return status_of(e);
}

int diffattn_v2_prefill_varlen(const void* q, const void* k, const void* v, const float* lambda, void* out,
                               const int32_t* cu_seqlens, int B, int max_seqlen, int total_tokens, int Hq, int Hkv,
                               int D, int causal, da2_stream_t stream) {
  if (B < 0 || max_seqlen < 0 || total_tokens < 0 || D <= 0 || !heads_ok(Hq, Hkv)) return DA2_ERR_INVALID;
  if (causal != 0 && causal != 1) return DA2_ERR_INVALID;
  if (B == 0 || max_seqlen == 0 || total_tokens == 0) return DA2_OK;
  if (!q || !k || !v || !lambda || !out || !cu_seqlens) return DA2_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(lambda) || !aligned16(out) ||
      !aligned16(cu_seqlens))
    return DA2_ERR_INVALID;
  if (D != 128) return DA2_ERR_UNSUPPORTED;
  if ((max_seqlen + 127) / 128 > 65535) return DA2_ERR_UNSUPPORTED;
  int* err = nullptr;
  cudaError_t e = device_error_ptr(&err);
  if (e != cudaSuccess) return DA2_ERR_CUDA;
  CUtensorMap tq, tk, tv, tkh;  // the packed tokens as one batch of total_tokens rows
  if (encode_bshd(&tq, q, D, Hq, total_tokens, 1, 64, 128) != cudaSuccess) return DA2_ERR_CUDA;
  if (encode_bshd(&tk, k, D, Hkv, total_tokens, 1, 64, 128) != cudaSuccess) return DA2_ERR_CUDA;
  if (encode_bshd(&tv, v, D, Hkv, total_tokens, 1, 64, 128) != cudaSuccess) return DA2_ERR_CUDA;
  if (encode_bshd(&tkh, k, D, Hkv, total_tokens, 1, 64, 64) != cudaSuccess) return DA2_ERR_CUDA;
  CUtensorMap to;
  if (da2::encode_out_bf16(&to, out, D, Hq / 2, total_tokens, 1) != cudaSuccess) return DA2_ERR_CUDA;
  e = da2::launch_prefill(tq, tk, tv, &tkh, to, lambda, static_cast<__nv_bfloat16*>(out), err, B, max_seqlen, Hq, Hkv, causal,
                          0, cu_seqlens, reinterpret_cast<cudaStream_t>(stream));
  return status_of(e);
}

int diffattn_v2_prefill_varlen_window(const void* q, const void* k, const void* v, const float* lambda, void* out,
                                      const int32_t* cu_seqlens, int B, int max_seqlen, int total_tokens, int Hq,
                                      int Hkv, int D, int window, da2_stream_t stream) {
  if (B < 0 || max_seqlen < 0 || total_tokens < 0 || D <= 0 || !heads_ok(Hq, Hkv) || window < 1) return DA2_ERR_INVALID;
  if (B == 0 || max_seqlen == 0 || total_tokens == 0) return DA2_OK;
  if (!q || !k || !v || !lambda || !out || !cu_seqlens) return DA2_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(lambda) || !aligned16(out) ||
      !aligned16(cu_seqlens))
    return DA2_ERR_INVALID;
  if (D != 128) return DA2_ERR_UNSUPPORTED;
  if ((max_seqlen + 127) / 128 > 65535) return DA2_ERR_UNSUPPORTED;
  int* err = nullptr;
  cudaError_t e = device_error_ptr(&err);
  if (e != cudaSuccess) return DA2_ERR_CUDA;
  CUtensorMap tq, tk, tv, tkh;  // the packed tokens as one batch of total_tokens rows
  if (encode_bshd(&tq, q, D, Hq, total_tokens, 1, 64, 128) != cudaSuccess) return DA2_ERR_CUDA;
  if (encode_bshd(&tk, k, D, Hkv, total_tokens, 1, 64, 128) != cudaSuccess) return DA2_ERR_CUDA;
  if (encode_bshd(&tv, v, D, Hkv, total_tokens, 1, 64, 128) != cudaSuccess) return DA2_ERR_CUDA;
  if (encode_bshd(&tkh, k, D, Hkv, total_tokens, 1, 64, 64) != cudaSuccess) return DA2_ERR_CUDA;
  CUtensorMap to;
  if (da2::encode_out_bf16(&to, out, D, Hq / 2, total_tokens, 1) != cudaSuccess) return DA2_ERR_CUDA;
  // a window of max_seqlen or more keys is the plain causal mask for every sequence
  e = da2::launch_prefill(tq, tk, tv, &tkh, to, lambda, static_cast<__nv_bfloat16*>(out), err, B, max_seqlen, Hq, Hkv,
                          1, window >= max_seqlen ? 0 : window, cu_seqlens, reinterpret_cast<cudaStream_t>(stream));
  return status_of(e);
}

int diffattn_v2_prefill_fused_lambda(const void* q, const void* k, const void* v, const void* x,
                                     const void* w_lambda_t, const float* bias, void* out, float* lambda_out, int B,
                                     int S, int Hq, int Hkv, int D, int d_model, int causal, da2_stream_t stream) {
  if (B < 0 || S < 0 || D <= 0 || !heads_ok(Hq, Hkv) || d_model <= 0 || (d_model % 8) != 0) return DA2_ERR_INVALID;
  if (causal != 0 && causal != 1) return DA2_ERR_INVALID;
  if (B == 0 || S == 0) return DA2_OK;
  if (!q || !k || !v || !x || !w_lambda_t || !out) return DA2_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(x) || !aligned16(w_lambda_t) || !aligned16(out) ||
      (bias && !aligned16(bias)) || (lambda_out && !aligned16(lambda_out)))
    return DA2_ERR_INVALID;
  if (D != 128) return DA2_ERR_UNSUPPORTED;
  if ((S + 127) / 128 > 65535) return DA2_ERR_UNSUPPORTED;
  int* err = nullptr;
  cudaError_t e = device_error_ptr(&err);
  if (e != cudaSuccess) return DA2_ERR_CUDA;
  CUtensorMap tq, tk, tv, to;
  if (encode_bshd(&tq, q, D, Hq, S, B, 64, 128) != cudaSuccess) return DA2_ERR_CUDA;
  if (encode_bshd(&tk, k, D, Hkv, S, B, 64, 128) != cudaSuccess) return DA2_ERR_CUDA;
  if (encode_bshd(&tv, v, D, Hkv, S, B, 64, 128) != cudaSuccess) return DA2_ERR_CUDA;
  if (da2::encode_out_bf16(&to, out, D, Hq / 2, S, B) != cudaSuccess) return DA2_ERR_CUDA;
  e = da2::launch_prefill_lambda_fused(tq, tk, tv, to, static_cast<const __nv_bfloat16*>(x),
                                       static_cast<const __nv_bfloat16*>(w_lambda_t), bias, lambda_out, d_model,
                                       static_cast<__nv_bfloat16*>(out), err, B, S, Hq, Hkv, causal,
                                       reinterpret_cast<cudaStream_t>(stream));
  return status_of(e);
}

int diffattn_v2_prefill_f32(const float* q, const float* k, const float* v, const float* lambda, float* out, int B,
                            int S, int Hq, int Hkv, int D, int causal, da2_stream_t stream) {
  if (B < 0 || S < 0 || D <= 0 || !heads_ok(Hq, Hkv)) return DA2_ERR_INVALID;
  if (causal != 0 && causal != 1) return DA2_ERR_INVALID;
  if (B == 0 || S == 0) return DA2_OK;
  if (!q || !k || !v || !lambda || !out) return DA2_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(lambda) || !aligned16(out))
    return DA2_ERR_INVALID;
  if (D != 64 && D != 128) return DA2_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * (Hq / 2) > 65535) return DA2_ERR_UNSUPPORTED;
  return status_of(da2::launch_prefill_f32(q, k, v, lambda, out, B, S, Hq, Hkv, D, causal,
                                           reinterpret_cast<cudaStream_t>(stream)));
}

int diffattn_v2_prefill_train(const void* q, const void* k, const void* v, const float* lambda, void* out,
                              void* o_branch, float* lse, int B, int S, int Hq, int Hkv, int D, int causal,
                              da2_stream_t stream) {
  if (B < 0 || S < 0 || D <= 0 || !heads_ok(Hq, Hkv)) return DA2_ERR_INVALID;
  if (causal != 0 && causal != 1) return DA2_ERR_INVALID;
  if (B == 0 || S == 0) return DA2_OK;
  if (!q || !k || !v || !lambda || !out || !o_branch || !lse) return DA2_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(lambda) || !aligned16(out) ||
      !aligned16(o_branch) || !aligned16(lse))
    return DA2_ERR_INVALID;
  if (D != 128) return DA2_ERR_UNSUPPORTED;
  if ((S + 127) / 128 > 65535) return DA2_ERR_UNSUPPORTED;
  int* err = nullptr;
  cudaError_t e = device_error_ptr(&err);
  if (e != cudaSuccess) return DA2_ERR_CUDA;
  CUtensorMap tq, tk, tv, tkh;
  if (encode_bshd(&tq, q, D, Hq, S, B, 64, 128) != cudaSuccess) return DA2_ERR_CUDA;
  if (encode_bshd(&tk, k, D, Hkv, S, B, 64, 128) != cudaSuccess) return DA2_ERR_CUDA;
  if (encode_bshd(&tv, v, D, Hkv, S, B, 64, 128) != cudaSuccess) return DA2_ERR_CUDA;
  if (encode_bshd(&tkh, k, D, Hkv, S, B, 64, 64) != cudaSuccess) return DA2_ERR_CUDA;
  CUtensorMap to;
  if (da2::encode_out_bf16(&to, out, D, Hq / 2, S, B) != cudaSuccess) return DA2_ERR_CUDA;
  e = da2::launch_prefill(tq, tk, tv, &tkh, to, lambda, static_cast<__nv_bfloat16*>(out), err, B, S, Hq, Hkv, causal, 0,
                          nullptr, reinterpret_cast<cudaStream_t>(stream), static_cast<__nv_bfloat16*>(o_branch),
                          lse);
  return status_of(e);
}

size_t diffattn_v2_backward_workspace_size(int B, int S, int Hq) {
  if (B <= 0 || S <= 0 || Hq <= 0 || (Hq % 2) != 0) return 0;
  return da2::backward_stats_bytes(B, S, Hq);
}

namespace {

// The [B,S] backward: causal 0/1, window > 0 only with causal (window >= S: plain causal).
int backward_bshd(const void* q, const void* k, const void* v, const float* lambda, const void* o_branch,
                  const float* lse, const void* dout, void* dq, void* dk, void* dv, float* dlambda, int B, int S,
                  int Hq, int Hkv, int D, int causal, int window, void* workspace, size_t workspace_bytes,
                  da2_stream_t stream) {
  if (B < 0 || S < 0 || D <= 0 || !heads_ok(Hq, Hkv)) return DA2_ERR_INVALID;
  if (causal != 0 && causal != 1) return DA2_ERR_INVALID;
  if (B == 0 || S == 0) return DA2_OK;
  const void* ptrs[] = {q, k, v, lambda, o_branch, lse, dout, dq, dk, dv, dlambda, workspace};
  for (const void* ptr : ptrs)
    if (!ptr || !aligned16(ptr)) return DA2_ERR_INVALID;
  if (workspace_bytes < diffattn_v2_backward_workspace_size(B, S, Hq)) return DA2_ERR_INVALID;
  if (D != 128) return DA2_ERR_UNSUPPORTED;
  // grid limits: 128-row tiles on grid y; the preprocess runs 4 (token, pair) warps per CTA
  if ((S + 127) / 128 > 65535) return DA2_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * ((S + 127) / 128 * 128) * (Hq / 2) > 4LL * 2147483647LL) return DA2_ERR_UNSUPPORTED;
  int* err = nullptr;
  if (device_error_ptr(&err) != cudaSuccess) return DA2_ERR_CUDA;
  CUtensorMap q64, q128, o64, o128, k64, k128, v64, v128;
  if (encode_bshd(&q64, q, D, Hq, S, B, 64, 64) != cudaSuccess || encode_bshd(&q128, q, D, Hq, S, B, 64, 128) != cudaSuccess ||
      encode_bshd(&o64, dout, D, Hq / 2, S, B, 64, 64) != cudaSuccess ||
      encode_bshd(&o128, dout, D, Hq / 2, S, B, 64, 128) != cudaSuccess ||
      encode_bshd(&k64, k, D, Hkv, S, B, 64, 64) != cudaSuccess || encode_bshd(&k128, k, D, Hkv, S, B, 64, 128) != cudaSuccess ||
      encode_bshd(&v64, v, D, Hkv, S, B, 64, 64) != cudaSuccess || encode_bshd(&v128, v, D, Hkv, S, B, 64, 128) != cudaSuccess)
    return DA2_ERR_CUDA;
  using bf = __nv_bfloat16;
  return status_of(da2::launch_backward_sm100(
      q64, q128, o64, o128, k64, k128, v64, v128, lambda, static_cast<const bf*>(o_branch), lse,
      static_cast<const bf*>(dout), static_cast<bf*>(dq), static_cast<bf*>(dk), static_cast<bf*>(dv), dlambda,
      static_cast<float*>(workspace), err, B, S, Hq, Hkv, causal, reinterpret_cast<cudaStream_t>(stream), nullptr, 0,
      window));
}

}  // namespace

int diffattn_v2_backward(const void* q, const void* k, const void* v, const float* lambda, const void* o_branch,
                         const float* lse, const void* dout, void* dq, void* dk, void* dv, float* dlambda, int B,
                         int S, int Hq, int Hkv, int D, int causal, void* workspace, size_t workspace_bytes,
                         da2_stream_t stream) {
  return backward_bshd(q, k, v, lambda, o_branch, lse, dout, dq, dk, dv, dlambda, B, S, Hq, Hkv, D, causal, 0,
                       workspace, workspace_bytes, stream);
}

int diffattn_v2_prefill_window_train(const void* q, const void* k, const void* v, const float* lambda, void* out,
                                     void* o_branch, float* lse, int B, int S, int Hq, int Hkv, int D, int window,
                                     da2_stream_t stream) {
  if (B < 0 || S < 0 || D <= 0 || !heads_ok(Hq, Hkv) || window < 1) return DA2_ERR_INVALID;
  if (B == 0 || S == 0) return DA2_OK;
  const void* ptrs[] = {q, k, v, lambda, out, o_branch, lse};
  for (const void* ptr : ptrs)
    if (!ptr || !aligned16(ptr)) return DA2_ERR_INVALID;
  if (D != 128) return DA2_ERR_UNSUPPORTED;
  if ((S + 127) / 128 > 65535) return DA2_ERR_UNSUPPORTED;
  int* err = nullptr;
  cudaError_t e = device_error_ptr(&err);
  if (e != cudaSuccess) return DA2_ERR_CUDA;
  CUtensorMap tq, tk, tv, tkh;
  if (encode_bshd(&tq, q, D, Hq, S, B, 64, 128) != cudaSuccess) return DA2_ERR_CUDA;
  if (encode_bshd(&tk, k, D, Hkv, S, B, 64, 128) != cudaSuccess) return DA2_ERR_CUDA;
  if (encode_bshd(&tv, v, D, Hkv, S, B, 64, 128) != cudaSuccess) return DA2_ERR_CUDA;
  if (encode_bshd(&tkh, k, D, Hkv, S, B, 64, 64) != cudaSuccess) return DA2_ERR_CUDA;
  CUtensorMap to;
  if (da2::encode_out_bf16(&to, out, D, Hq / 2, S, B) != cudaSuccess) return DA2_ERR_CUDA;
  // a window of S or more keys is the plain causal mask
  e = da2::launch_prefill(tq, tk, tv, &tkh, to, lambda, static_cast<__nv_bfloat16*>(out), err, B, S, Hq, Hkv, 1,
                          window >= S ? 0 : window, nullptr, reinterpret_cast<cudaStream_t>(stream),
                          static_cast<__nv_bfloat16*>(o_branch), lse);
  return status_of(e);
}

int diffattn_v2_backward_window(const void* q, const void* k, const void* v, const float* lambda,
                                const void* o_branch, const float* lse, const void* dout, void* dq, void* dk,
                                void* dv, float* dlambda, int B, int S, int Hq, int Hkv, int D, int window,
                                void* workspace, size_t workspace_bytes, da2_stream_t stream) {
  if (window < 1) return DA2_ERR_INVALID;
  return backward_bshd(q, k, v, lambda, o_branch, lse, dout, dq, dk, dv, dlambda, B, S, Hq, Hkv, D, 1,
                       window >= S ? 0 : window, workspace, workspace_bytes, stream);
}

namespace {

// Training forward of packed sequences; window > 0 (causal only) applies inside each sequence.
int prefill_varlen_train(const void* q, const void* k, const void* v, const float* lambda, void* out, void* o_branch,
                         float* lse, const int32_t* cu_seqlens, int B, int max_seqlen, int total_tokens, int Hq,
                         int Hkv, int D, int causal, int window, da2_stream_t stream) {
  if (B < 0 || max_seqlen < 0 || total_tokens < 0 || D <= 0 || !heads_ok(Hq, Hkv)) return DA2_ERR_INVALID;
  if (causal != 0 && causal != 1) return DA2_ERR_INVALID;
  if (B == 0 || max_seqlen == 0 || total_tokens == 0) return DA2_OK;
  const void* ptrs[] = {q, k, v, lambda, out, o_branch, lse, cu_seqlens};
  for (const void* ptr : ptrs)
    if (!ptr || !aligned16(ptr)) return DA2_ERR_INVALID;
  if (D != 128) return DA2_ERR_UNSUPPORTED;
  if ((max_seqlen + 127) / 128 > 65535) return DA2_ERR_UNSUPPORTED;
  int* err = nullptr;
  cudaError_t e = device_error_ptr(&err);
  if (e != cudaSuccess) return DA2_ERR_CUDA;
  CUtensorMap tq, tk, tv, tkh;  // the packed tokens as one batch of total_tokens rows
  if (encode_bshd(&tq, q, D, Hq, total_tokens, 1, 64, 128) != cudaSuccess) return DA2_ERR_CUDA;
  if (encode_bshd(&tk, k, D, Hkv, total_tokens, 1, 64, 128) != cudaSuccess) return DA2_ERR_CUDA;
  if (encode_bshd(&tv, v, D, Hkv, total_tokens, 1, 64, 128) != cudaSuccess) return DA2_ERR_CUDA;
  if (encode_bshd(&tkh, k, D, Hkv, total_tokens, 1, 64, 64) != cudaSuccess) return DA2_ERR_CUDA;
  CUtensorMap to;
  if (da2::encode_out_bf16(&to, out, D, Hq / 2, total_tokens, 1) != cudaSuccess) return DA2_ERR_CUDA;
  e = da2::launch_prefill(tq, tk, tv, &tkh, to, lambda, static_cast<__nv_bfloat16*>(out), err, B, max_seqlen, Hq, Hkv, causal,
                          window, cu_seqlens, reinterpret_cast<cudaStream_t>(stream),
                          static_cast<__nv_bfloat16*>(o_branch), lse);
  return status_of(e);
}

}  // namespace

int diffattn_v2_prefill_varlen_train(const void* q, const void* k, const void* v, const float* lambda, void* out,
                                     void* o_branch, float* lse, const int32_t* cu_seqlens, int B, int max_seqlen,
                                     int total_tokens, int Hq, int Hkv, int D, int causal, da2_stream_t stream) {
  return prefill_varlen_train(q, k, v, lambda, out, o_branch, lse, cu_seqlens, B, max_seqlen, total_tokens, Hq, Hkv,
                              D, causal, 0, stream);
}

int diffattn_v2_prefill_varlen_window_train(const void* q, const void* k, const void* v, const float* lambda,
                                            void* out, void* o_branch, float* lse, const int32_t* cu_seqlens, int B,
                                            int max_seqlen, int total_tokens, int Hq, int Hkv, int D, int window,
                                            da2_stream_t stream) {
  if (window < 1) return DA2_ERR_INVALID;
  // a window of max_seqlen or more keys is the plain causal mask for every sequence
  return prefill_varlen_train(q, k, v, lambda, out, o_branch, lse, cu_seqlens, B, max_seqlen, total_tokens, Hq, Hkv,
                              D, 1, window >= max_seqlen ? 0 : window, stream);
}

size_t diffattn_v2_backward_varlen_workspace_size(int B, int total_tokens, int Hq) {
  if (B <= 0 || total_tokens <= 0 || Hq <= 0 || (Hq % 2) != 0) return 0;
  return da2::backward_varlen_workspace_bytes(B, total_tokens, Hq);
}

namespace {

// Backward of the packed-sequence prefill; window > 0 (causal only) inside each sequence.
int backward_varlen(const void* q, const void* k, const void* v, const float* lambda, const void* o_branch,
                    const float* lse, const void* dout, void* dq, void* dk, void* dv, float* dlambda,
                    const int32_t* cu_seqlens, int B, int max_seqlen, int total_tokens, int Hq, int Hkv, int D,
                    int causal, int window, void* workspace, size_t workspace_bytes, da2_stream_t stream) {
  if (B < 0 || max_seqlen < 0 || total_tokens < 0 || D <= 0 || !heads_ok(Hq, Hkv)) return DA2_ERR_INVALID;
  if (causal != 0 && causal != 1) return DA2_ERR_INVALID;
  if (B == 0 || max_seqlen == 0 || total_tokens == 0) return DA2_OK;
  const void* ptrs[] = {q, k, v, lambda, o_branch, lse, dout, dq, dk, dv, dlambda, cu_seqlens, workspace};
  for (const void* ptr : ptrs)
    if (!ptr || !aligned16(ptr)) return DA2_ERR_INVALID;
  if (workspace_bytes < diffattn_v2_backward_varlen_workspace_size(B, total_tokens, Hq)) return DA2_ERR_INVALID;
  if (D != 128) return DA2_ERR_UNSUPPORTED;
  // grid limits: 128-row tiles on grid y; the preprocess runs 4 (row, pair) warps per CTA
  if ((max_seqlen + 127) / 128 > 65535) return DA2_ERR_UNSUPPORTED;
  if ((static_cast<long long>(total_tokens) + 128LL * B + 128) * (Hq / 2) > 4LL * 2147483647LL) return DA2_ERR_UNSUPPORTED;
  int* err = nullptr;
  if (device_error_ptr(&err) != cudaSuccess) return DA2_ERR_CUDA;
  const int T = total_tokens;
  CUtensorMap q64, q128, o64, o128, k64, k128, v64, v128;
  if (encode_bshd(&q64, q, D, Hq, T, 1, 64, 64) != cudaSuccess || encode_bshd(&q128, q, D, Hq, T, 1, 64, 128) != cudaSuccess ||
      encode_bshd(&o64, dout, D, Hq / 2, T, 1, 64, 64) != cudaSuccess ||
      encode_bshd(&o128, dout, D, Hq / 2, T, 1, 64, 128) != cudaSuccess ||
      encode_bshd(&k64, k, D, Hkv, T, 1, 64, 64) != cudaSuccess || encode_bshd(&k128, k, D, Hkv, T, 1, 64, 128) != cudaSuccess ||
      encode_bshd(&v64, v, D, Hkv, T, 1, 64, 64) != cudaSuccess || encode_bshd(&v128, v, D, Hkv, T, 1, 64, 128) != cudaSuccess)
    return DA2_ERR_CUDA;
  using bf = __nv_bfloat16;
  return status_of(da2::launch_backward_sm100(
      q64, q128, o64, o128, k64, k128, v64, v128, lambda, static_cast<const bf*>(o_branch), lse,
      static_cast<const bf*>(dout), static_cast<bf*>(dq), static_cast<bf*>(dk), static_cast<bf*>(dv), dlambda,
      static_cast<float*>(workspace), err, B, max_seqlen, Hq, Hkv, causal, reinterpret_cast<cudaStream_t>(stream),
      cu_seqlens, T, window));
}

}  // namespace

int diffattn_v2_backward_varlen(const void* q, const void* k, const void* v, const float* lambda,
                                const void* o_branch, const float* lse, const void* dout, void* dq, void* dk,
                                void* dv, float* dlambda, const int32_t* cu_seqlens, int B, int max_seqlen,
                                int total_tokens, int Hq, int Hkv, int D, int causal, void* workspace,
                                size_t workspace_bytes, da2_stream_t stream) {
  return backward_varlen(q, k, v, lambda, o_branch, lse, dout, dq, dk, dv, dlambda, cu_seqlens, B, max_seqlen,
                         total_tokens, Hq, Hkv, D, causal, 0, workspace, workspace_bytes, stream);
}

int diffattn_v2_backward_varlen_window(const void* q, const void* k, const void* v, const float* lambda,
                                       const void* o_branch, const float* lse, const void* dout, void* dq, void* dk,
                                       void* dv, float* dlambda, const int32_t* cu_seqlens, int B, int max_seqlen,
                                       int total_tokens, int Hq, int Hkv, int D, int window, void* workspace,
                                       size_t workspace_bytes, da2_stream_t stream) {
  if (window < 1) return DA2_ERR_INVALID;
  return backward_varlen(q, k, v, lambda, o_branch, lse, dout, dq, dk, dv, dlambda, cu_seqlens, B, max_seqlen,
                         total_tokens, Hq, Hkv, D, 1, window >= max_seqlen ? 0 : window, workspace, workspace_bytes,
                         stream);
}

size_t diffattn_v2_decode_workspace_size(int B, int Smax, int Hq, int Hkv, int D) {
  if (B <= 0 || Smax <= 0 || D <= 0 || !heads_ok(Hq, Hkv)) return 0;
  int split_len = 0, nsplit = 0;
  da2::decode_split_plan(B, Smax, Hkv, &split_len, &nsplit);
  return da2::decode_workspace_bytes(B, 1, Hq, Hkv, D, nsplit);
}

namespace {

// The bf16 decode over [B,Smax,Hkv,D] caches; window > 0: only the last `window` keys.
int decode_bshd(const void* q, const void* kcache, const void* vcache, const int32_t* seqlens, const float* lambda,
                void* out, int B, int Smax, int Hq, int Hkv, int D, int window, void* workspace,
                size_t workspace_bytes, da2_stream_t stream) {
  if (B < 0 || Smax <= 0 || D <= 0 || !heads_ok(Hq, Hkv) || window < 0) return DA2_ERR_INVALID;
  if (B == 0) return DA2_OK;
  if (!q || !kcache || !vcache || !seqlens || !lambda || !out || !workspace) return DA2_ERR_INVALID;
  if (!aligned16(q) || !aligned16(kcache) || !aligned16(vcache) || !aligned16(seqlens) || !aligned16(lambda) ||
      !aligned16(out) || !aligned16(workspace))
    return DA2_ERR_INVALID;
  if (workspace_bytes < diffattn_v2_decode_workspace_size(B, Smax, Hq, Hkv, D)) return DA2_ERR_INVALID;
  const int group = Hq / Hkv;
  if (D != 128 || !(group == 2 || group == 4 || group == 8 || group == 16)) return DA2_ERR_UNSUPPORTED;
  if (B > 65535 || Hkv > 65535) return DA2_ERR_UNSUPPORTED;
  int* err = nullptr;
  cudaError_t e = device_error_ptr(&err);
  if (e != cudaSuccess) return DA2_ERR_CUDA;
  int split_len = 0, nsplit = 0;
  da2::decode_split_plan_window(B, Smax, Hkv, window, &split_len, &nsplit);
  CUtensorMap tk, tv;
  if (encode_bshd(&tk, kcache, D, Hkv, Smax, B, 64, 64) != cudaSuccess) return DA2_ERR_CUDA;
  if (encode_bshd(&tv, vcache, D, Hkv, Smax, B, 64, 64) != cudaSuccess) return DA2_ERR_CUDA;
  const da2::DecodeWorkspace ws = da2::decode_workspace_layout(workspace, B, 1, Hq, D, nsplit);
  e = da2::launch_decode(tk, tv, static_cast<const __nv_bfloat16*>(q), seqlens, lambda,
                         static_cast<__nv_bfloat16*>(out), ws.o, ws.ml, ws.counters, err, B, Smax, Hq, Hkv, nsplit,
                         split_len, nullptr, 0, 0, 1, reinterpret_cast<cudaStream_t>(stream), window);
  return status_of(e);
}

}  // namespace

int diffattn_v2_decode(const void* q, const void* kcache, const void* vcache, const int32_t* seqlens,
                       const float* lambda, void* out, int B, int Smax, int Hq, int Hkv, int D, void* workspace,
                       size_t workspace_bytes, da2_stream_t stream) {
  return decode_bshd(q, kcache, vcache, seqlens, lambda, out, B, Smax, Hq, Hkv, D, 0, workspace, workspace_bytes,
                     stream);
}

int diffattn_v2_decode_window(const void* q, const void* kcache, const void* vcache, const int32_t* seqlens,
                              const float* lambda, void* out, int B, int Smax, int Hq, int Hkv, int D, int window,
                              void* workspace, size_t workspace_bytes, da2_stream_t stream) {
  if (window < 1) return DA2_ERR_INVALID;
  // a window of Smax or more keys sees every cached key
  return decode_bshd(q, kcache, vcache, seqlens, lambda, out, B, Smax, Hq, Hkv, D, window >= Smax ? 0 : window,
                     workspace, workspace_bytes, stream);
}

namespace {

// The bf16 decode over a paged cache; window > 0: only the last `window` keys.
int decode_paged(const void* q, const void* kpages, const void* vpages, const int32_t* block_table,
                 const int32_t* seqlens, const float* lambda, void* out, int B, int max_pages, int page_size,
                 int num_pages, int Hq, int Hkv, int D, int window, void* workspace, size_t workspace_bytes,
                 da2_stream_t stream) {
  if (B < 0 || max_pages <= 0 || num_pages <= 0 || D <= 0 || !heads_ok(Hq, Hkv) || window < 0) return DA2_ERR_INVALID;
  if (page_size < 8 || page_size > 4096 || (page_size & (page_size - 1)) != 0) return DA2_ERR_INVALID;
  if (static_cast<long long>(max_pages) * page_size > (1LL << 30)) return DA2_ERR_INVALID;
  if (B == 0) return DA2_OK;
  if (!q || !kpages || !vpages || !block_table || !seqlens || !lambda || !out || !workspace) return DA2_ERR_INVALID;
  if (!aligned16(q) || !aligned16(kpages) || !aligned16(vpages) || !aligned16(block_table) || !aligned16(seqlens) ||
      !aligned16(lambda) || !aligned16(out) || !aligned16(workspace))
    return DA2_ERR_INVALID;
  const int Smax = max_pages * page_size;
  if (workspace_bytes < diffattn_v2_decode_workspace_size(B, Smax, Hq, Hkv, D)) return DA2_ERR_INVALID;
  const int group = Hq / Hkv;
  if (D != 128 || !(group == 2 || group == 4 || group == 8 || group == 16)) return DA2_ERR_UNSUPPORTED;
  if (B > 65535 || Hkv > 65535) return DA2_ERR_UNSUPPORTED;
  int* err = nullptr;
  cudaError_t e = device_error_ptr(&err);
  if (e != cudaSuccess) return DA2_ERR_CUDA;
  if (window >= Smax) window = 0;
  int split_len = 0, nsplit = 0;
  da2::decode_split_plan_window(B, Smax, Hkv, window, &split_len, &nsplit);
  int page_shift = 0;
  while ((1 << page_shift) < page_size) ++page_shift;
  const uint32_t box = static_cast<uint32_t>(page_size < 64 ? page_size : 64);
  CUtensorMap tk, tv;  // pages as a [num_pages, page_size] batch of rows
  if (encode_bshd(&tk, kpages, D, Hkv, page_size, num_pages, 64, box) != cudaSuccess) return DA2_ERR_CUDA;
  if (encode_bshd(&tv, vpages, D, Hkv, page_size, num_pages, 64, box) != cudaSuccess) return DA2_ERR_CUDA;
  const da2::DecodeWorkspace ws = da2::decode_workspace_layout(workspace, B, 1, Hq, D, nsplit);
  e = da2::launch_decode(tk, tv, static_cast<const __nv_bfloat16*>(q), seqlens, lambda,
                         static_cast<__nv_bfloat16*>(out), ws.o, ws.ml, ws.counters, err, B, Smax, Hq, Hkv, nsplit,
                         split_len, block_table, max_pages, page_shift, 1, reinterpret_cast<cudaStream_t>(stream),
                         window);
  return status_of(e);
}

}  // namespace

int diffattn_v2_decode_paged(const void* q, const void* kpages, const void* vpages, const int32_t* block_table,
                             const int32_t* seqlens, const float* lambda, void* out, int B, int max_pages,
                             int page_size, int num_pages, int Hq, int Hkv, int D, void* workspace,
                             size_t workspace_bytes, da2_stream_t stream) {
  return decode_paged(q, kpages, vpages, block_table, seqlens, lambda, out, B, max_pages, page_size, num_pages, Hq,
                      Hkv, D, 0, workspace, workspace_bytes, stream);
}

int diffattn_v2_decode_paged_window(const void* q, const void* kpages, const void* vpages,
                                    const int32_t* block_table, const int32_t* seqlens, const float* lambda,
                                    void* out, int B, int max_pages, int page_size, int num_pages, int Hq, int Hkv,
                                    int D, int window, void* workspace, size_t workspace_bytes,
                                    da2_stream_t stream) {
  if (window < 1) return DA2_ERR_INVALID;
  return decode_paged(q, kpages, vpages, block_table, seqlens, lambda, out, B, max_pages, page_size, num_pages, Hq,
                      Hkv, D, window, workspace, workspace_bytes, stream);
}

size_t diffattn_v2_decode_multi_workspace_size(int B, int T, int Smax, int Hq, int Hkv, int D) {
  if (B <= 0 || T <= 0 || Smax <= 0 || D <= 0 || !heads_ok(Hq, Hkv)) return 0;
  int split_len = 0, nsplit = 0;
  da2::decode_split_plan(B, Smax, Hkv, &split_len, &nsplit);
  return da2::decode_workspace_bytes(B, T, Hq, Hkv, D, nsplit);
}

int diffattn_v2_decode_multi(const void* q, const void* kcache, const void* vcache, const int32_t* seqlens,
                             const float* lambda, void* out, int B, int T, int Smax, int Hq, int Hkv, int D,
                             void* workspace, size_t workspace_bytes, da2_stream_t stream) {
  if (B < 0 || T <= 0 || Smax <= 0 || D <= 0 || !heads_ok(Hq, Hkv)) return DA2_ERR_INVALID;
  if (B == 0) return DA2_OK;
  if (!q || !kcache || !vcache || !seqlens || !lambda || !out || !workspace) return DA2_ERR_INVALID;
  if (!aligned16(q) || !aligned16(kcache) || !aligned16(vcache) || !aligned16(seqlens) || !aligned16(lambda) ||
      !aligned16(out) || !aligned16(workspace))
    return DA2_ERR_INVALID;
  if (workspace_bytes < diffattn_v2_decode_multi_workspace_size(B, T, Smax, Hq, Hkv, D)) return DA2_ERR_INVALID;
  const int group = Hq / Hkv;
  if (D != 128 || !(group == 2 || group == 4 || group == 8 || group == 16) || T * group > 16)
    return DA2_ERR_UNSUPPORTED;
  if (B > 65535 || Hkv > 65535) return DA2_ERR_UNSUPPORTED;
  int* err = nullptr;
  cudaError_t e = device_error_ptr(&err);
  if (e != cudaSuccess) return DA2_ERR_CUDA;
  int split_len = 0, nsplit = 0;
  da2::decode_split_plan(B, Smax, Hkv, &split_len, &nsplit);
  CUtensorMap tk, tv;
  if (encode_bshd(&tk, kcache, D, Hkv, Smax, B, 64, 64) != cudaSuccess) return DA2_ERR_CUDA;
  if (encode_bshd(&tv, vcache, D, Hkv, Smax, B, 64, 64) != cudaSuccess) return DA2_ERR_CUDA;
  const da2::DecodeWorkspace ws = da2::decode_workspace_layout(workspace, B, T, Hq, D, nsplit);
  e = da2::launch_decode(tk, tv, static_cast<const __nv_bfloat16*>(q), seqlens, lambda,
                         static_cast<__nv_bfloat16*>(out), ws.o, ws.ml, ws.counters, err, B, Smax, Hq, Hkv, nsplit,
                         split_len,
                         nullptr, 0, 0, T, reinterpret_cast<cudaStream_t>(stream));
  return status_of(e);
}

int diffattn_v2_decode_f32(const float* q, const float* kcache, const float* vcache, const int32_t* seqlens,
                           const float* lambda, float* out, int B, int Smax, int Hq, int Hkv, int D,
                           da2_stream_t stream) {
  if (B < 0 || Smax <= 0 || D <= 0 || !heads_ok(Hq, Hkv)) return DA2_ERR_INVALID;
  if (B == 0) return DA2_OK;
  if (!q || !kcache || !vcache || !seqlens || !lambda || !out) return DA2_ERR_INVALID;
  if (!aligned16(q) || !aligned16(kcache) || !aligned16(vcache) || !aligned16(seqlens) || !aligned16(lambda) ||
      !aligned16(out))
    return DA2_ERR_INVALID;
  if (D != 64 && D != 128) return DA2_ERR_UNSUPPORTED;
  return status_of(da2::launch_decode_f32(q, kcache, vcache, seqlens, lambda, out, B, Smax, Hq, Hkv, D,
                                          reinterpret_cast<cudaStream_t>(stream)));
}

int diffattn_v2_lambda_v1(const float* lq1, const float* lk1, const float* lq2, const float* lk2, float lambda_init,
                          int n_pairs, int d, int rows, float* lambda_out, da2_stream_t stream) {
  if (n_pairs <= 0 || d <= 0 || rows < 0) return DA2_ERR_INVALID;
  if (rows == 0) return DA2_OK;
  if (!lq1 || !lk1 || !lq2 || !lk2 || !lambda_out) return DA2_ERR_INVALID;
  if (!aligned16(lq1) || !aligned16(lk1) || !aligned16(lq2) || !aligned16(lk2) || !aligned16(lambda_out))
    return DA2_ERR_INVALID;
  return status_of(da2::launch_lambda_v1(lq1, lk1, lq2, lk2, lambda_init, n_pairs, d, rows, lambda_out,
                                         reinterpret_cast<cudaStream_t>(stream)));
}

int diffattn_v2_lambda_v2(const void* x, const void* w_lambda, const float* bias, int T, int d_model, int n_pairs,
                          float* lambda_out, da2_stream_t stream) {
  if (T < 0 || d_model <= 0 || n_pairs <= 0) return DA2_ERR_INVALID;
  if (T == 0) return DA2_OK;
  if (!x || !w_lambda || !lambda_out) return DA2_ERR_INVALID;
  if (!aligned16(x) || !aligned16(w_lambda) || !aligned16(lambda_out) || (bias && !aligned16(bias)))
    return DA2_ERR_INVALID;
  if (d_model % 64 != 0 || n_pairs % 8 != 0 || n_pairs > 64) return DA2_ERR_UNSUPPORTED;
  int* err = nullptr;
  if (device_error_ptr(&err) != cudaSuccess) return DA2_ERR_CUDA;
  CUtensorMap tx, tw;
  if (da2::encode_2d_bf16(&tx, x, d_model, T, static_cast<uint64_t>(d_model) * 2, 64, 128) != cudaSuccess)
    return DA2_ERR_CUDA;
  if (da2::encode_2d_bf16(&tw, w_lambda, n_pairs, d_model, static_cast<uint64_t>(n_pairs) * 2, 64, 64) != cudaSuccess)
    return DA2_ERR_CUDA;
  return status_of(da2::launch_lambda_v2(tx, tw, bias, T, d_model, n_pairs, lambda_out, err,
                                         reinterpret_cast<cudaStream_t>(stream)));
}

int diffattn_v2_device_error(int* code, da2_stream_t stream) {
  cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return DA2_ERR_CUDA;
  int* err = nullptr;
  e = device_error_ptr(&err);
  if (e != cudaSuccess) return DA2_ERR_CUDA;
  int h = 0;
  e = cudaMemcpy(&h, err, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return DA2_ERR_CUDA;
  if (h != 0) {
    const int zero = 0;
    e = cudaMemcpy(err, &zero, sizeof(int), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return DA2_ERR_CUDA;
  }
  if (code) *code = h;
  return h ? DA2_ERR_DEVICE : DA2_OK;
}

}  // extern "C"
