// internal.h -- host-side launchers shared between the C ABI (api.cu) and the kernel files.
// Not installed; the public interface is include/diffattn_v2.h.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace da2 {

// bf16 prefill on tcgen05 (D = 128); window > 0 (causal only) limits query i to keys
// i-window+1 .. i. With cu_seqlens (device, B+1 entries) the tensors hold B packed sequences
// as one [1,T] batch and S is the longest sequence. Tensor maps: Q over [B,S,Hq,D], K/V over [B,S,Hkv,D],
// boxes of 64 (d) x 1 (head) x 128 (rows) x 1, 128-byte swizzle; tmKh (optional) over K with
// boxes of 64 (d) x 1 x 64 (rows) x 1, for the CTA-pair form (GQA groups of a multiple of 4);
// tmO over out [B,S,Hq/2,D] (with cu_seqlens [1,T,Hq/2,D]) from encode_out_bf16.
cudaError_t launch_prefill(const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV,
                           const CUtensorMap* tmKh, const CUtensorMap& tmO, const float* lambda, __nv_bfloat16* out, int* err, int B, int S,
                           int Hq, int Hkv, int causal, int window, const int* cu_seqlens, cudaStream_t stream,
                           __nv_bfloat16* o_branch = nullptr, float* lse = nullptr);

// The [B,S] bf16 prefill with the V2 lambda computed in the kernel:
// lambda[t, p] = sigmoid(x[t] . w_t[p] + bias[p]) with x [B*S, d_model] and w_t [Hq/2, d_model]
// bf16 (d_model a multiple of 8), bias fp32 [Hq/2] or null; lambda_out (fp32 [B*S, Hq/2]) gets
// a copy when not null. Tensor maps as for launch_prefill.
cudaError_t launch_prefill_lambda_fused(const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV,
                                        const CUtensorMap& tmO, const __nv_bfloat16* x, const __nv_bfloat16* w_t,
                                        const float* bias, float* lambda_out, int d_model, __nv_bfloat16* out,
                                        int* err, int B, int S, int Hq, int Hkv, int causal, cudaStream_t stream);

// tcgen05 backward of the bf16 prefill (D = 128): preprocess into the workspace (row terms;
// backward_stats_bytes, or backward_varlen_workspace_bytes with packed sequences), then the
// dK/dV and dQ tile kernels. Tensor maps over q [B,S,Hq,D], dout [B,S,Hq/2,D], k and v
// [B,S,Hkv,D] with 64- and 128-row boxes (64 d x 1 head). With cu_seqlens (device, B+1
// entries) the tensors hold B packed sequences as one [1,T] batch (T = total_tokens) and S
// is the longest sequence. window > 0 (causal only): query i saw keys i-window+1 .. i.
size_t backward_stats_bytes(int B, int S, int Hq);
size_t backward_varlen_workspace_bytes(int B, int T, int Hq);
cudaError_t launch_backward_sm100(const CUtensorMap& tmQ64, const CUtensorMap& tmQ128, const CUtensorMap& tmO64,
                                  const CUtensorMap& tmO128, const CUtensorMap& tmK64, const CUtensorMap& tmK128,
                                  const CUtensorMap& tmV64, const CUtensorMap& tmV128, const float* lambda,
                                  const __nv_bfloat16* o_branch, const float* lse, const __nv_bfloat16* dout,
                                  __nv_bfloat16* dq, __nv_bfloat16* dk, __nv_bfloat16* dv, float* dlambda,
                                  float* workspace, int* err, int B, int S, int Hq, int Hkv, int causal,
                                  cudaStream_t stream, const int32_t* cu_seqlens = nullptr, int total_tokens = 0,
                                  int window = 0);

// bf16 decode (D = 128): split kernel + combine. Tensor maps over the caches [B,Smax,Hkv,D],
// boxes of 64 (d) x 1 x 64 (tokens) x 1, 128-byte swizzle. With block_table the maps cover
// pages [num_pages, 1 << page_shift, Hkv, D] with boxes of min(page_size, 64) tokens and
// Smax = max_pages << page_shift. T new tokens per sequence (q [B,T,Hq,D]); T * Hq/Hkv <= 16.
cudaError_t launch_decode(const CUtensorMap& tmK, const CUtensorMap& tmV, const __nv_bfloat16* q,
                          const int32_t* seqlens, const float* lambda, __nv_bfloat16* out, float* ws_o,
                          float* ws_ml, int* counters, int* err, int B, int Smax, int Hq, int Hkv, int nsplit,
                          int split_len, const int32_t* block_table, int max_pages, int page_shift, int T,
                          cudaStream_t stream, int window = 0);

// Tokens per split and number of splits of the bf16 decode for these sizes.
void decode_split_plan(int B, int Smax, int Hkv, int* split_len, int* nsplit);
// The same for a sliding-window decode (window > 0): splits over the window's span when that
// needs no more splits than the plan for Smax (the workspace is sized by that plan).
void decode_split_plan_window(int B, int Smax, int Hkv, int window, int* split_len, int* nsplit);

// The bf16 decode's workspace, in this order: fp32 partial outputs O [rows, D], fp32 (m, l)
// [rows, 2], then one int split counter per (b, KV head), padded to 16 bytes; rows =
// B * T * Hq * nsplit (T new tokens per sequence). Every entry point that hands the split
// kernel a workspace (caller-provided or the library's own array) lays it out through these.
struct DecodeWorkspace {
  float* o;
  float* ml;
  int* counters;
};
size_t decode_workspace_bytes(int B, int T, int Hq, int Hkv, int D, int nsplit);
DecodeWorkspace decode_workspace_layout(void* base, int B, int T, int Hq, int D, int nsplit);

// fp32 CUDA-core paths (D in {64, 128}).
cudaError_t launch_prefill_f32(const float* q, const float* k, const float* v, const float* lambda, float* out,
                               int B, int S, int Hq, int Hkv, int D, int causal, cudaStream_t stream);
cudaError_t launch_decode_f32(const float* q, const float* kc, const float* vc, const int32_t* seqlens,
                              const float* lambda, float* out, int B, int Smax, int Hq, int Hkv, int D,
                              cudaStream_t stream);

// V1 lambda, broadcast to `rows` rows.
cudaError_t launch_lambda_v1(const float* lq1, const float* lk1, const float* lq2, const float* lk2,
                             float lambda_init, int n_pairs, int d, int rows, float* out, cudaStream_t stream);

// Address of the device error word on the current device.
cudaError_t device_error_word(int** out);

// 4-D bf16 tensor map over a row-major [B,S,H,D] array, box {box0, 1, box2, 1}, 128-byte swizzle.
cudaError_t encode_bshd_bf16(CUtensorMap* map, const void* base, uint64_t D, uint64_t H, uint64_t S, uint64_t B,
                             uint32_t box0, uint32_t box2);

// 4-D bf16 tensor map for the prefill's output stores: [B,S,H,D] (H = Hq/2 pairs), box
// {32, 1, 32, 1} (32 columns of 32 rows of one pair), 64-byte swizzle.
cudaError_t encode_out_bf16(CUtensorMap* map, void* base, uint64_t D, uint64_t H, uint64_t S, uint64_t B);

// V2 lambda projection sigmoid(x W + bias) on tcgen05: tmX over x [T, d_model] bf16 with
// boxes of 64 (d_model) x 128 (tokens), tmW over W [d_model, n_pairs] bf16 with boxes of 64
// (pair columns; those past n_pairs read as zeros) x 64 (d_model), both 128-byte swizzled;
// bias fp32 [n_pairs] or null; d_model % 64 == 0, n_pairs % 8 == 0 and <= 64.
cudaError_t launch_lambda_v2(const CUtensorMap& tmX, const CUtensorMap& tmW, const float* bias, int T, int d_model,
                             int n_pairs, float* out, int* err, cudaStream_t stream);

// 2-D bf16 tensor map over a row-major [rows, cols] array with row stride `row_bytes`, box
// {box_cols, box_rows}, 128-byte swizzle, out-of-range elements read as zero.
cudaError_t encode_2d_bf16(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows, uint64_t row_bytes,
                           uint32_t box_cols, uint32_t box_rows);

}  // namespace da2
