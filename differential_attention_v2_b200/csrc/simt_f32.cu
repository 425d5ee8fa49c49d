// simt_f32.cu -- fp32 DiffAttn V2 prefill and decode on the CUDA cores.
//
// For callers that need results within ~1e-5 of exact: no tensor cores (TF32 could not
// reach that), accurate expf, fp32 accumulation. The operator is the one of the
// "Differential Attention (V2)" lesson, "The differential concept" (A1, A2 and
// DiffAttn = (A1 - lambda A2) V), with the causal mask of the "Attention variants" lesson,
// Step 1, and the V2 head pairing (adjacent heads of one GQA group share K/V).
//
// One warp computes one output row of one pair (both branches): lanes take 32 keys at a
// time for the scores, then the warp accumulates p_j * v_j with lane l owning output
// dimensions l, l+32, ... A running max and sum per branch make it a single pass over the
// keys (online softmax, natural-log domain).

#include "internal.h"

namespace da2 {
namespace simt {

template <int D>
__device__ __forceinline__ void diff_row_f32(const float* __restrict__ q1, const float* __restrict__ q2,
                                             const float* __restrict__ kbase, const float* __restrict__ vbase,
                                             int row_stride, int n_keys, float lam, float* __restrict__ out,
                                             float* __restrict__ sq /* 2*D floats of this warp */) {
  constexpr int U = D / 32;
  const int lane = threadIdx.x & 31;
  const float scale = rsqrtf(static_cast<float>(D));
#pragma unroll
  for (int u = 0; u < U; ++u) {
    sq[lane + 32 * u] = q1[lane + 32 * u];
    sq[D + lane + 32 * u] = q2[lane + 32 * u];
  }
  __syncwarp();
  float m1 = -INFINITY, m2 = -INFINITY, l1 = 0.f, l2 = 0.f;
  float acc1[U], acc2[U];
#pragma unroll
  for (int u = 0; u < U; ++u) acc1[u] = acc2[u] = 0.f;

  for (int j0 = 0; j0 < n_keys; j0 += 32) {
    const int j = j0 + lane;
    float s1 = -INFINITY, s2 = -INFINITY;
    if (j < n_keys) {
      const float4* kr = reinterpret_cast<const float4*>(kbase + static_cast<size_t>(j) * row_stride);
      float d1 = 0.f, d2 = 0.f;
#pragma unroll 8
      for (int c = 0; c < D / 4; ++c) {
        const float4 kv = __ldg(kr + c);
        d1 = fmaf(sq[4 * c + 0], kv.x, d1);
        d1 = fmaf(sq[4 * c + 1], kv.y, d1);
        d1 = fmaf(sq[4 * c + 2], kv.z, d1);
        d1 = fmaf(sq[4 * c + 3], kv.w, d1);
        d2 = fmaf(sq[D + 4 * c + 0], kv.x, d2);
        d2 = fmaf(sq[D + 4 * c + 1], kv.y, d2);
        d2 = fmaf(sq[D + 4 * c + 2], kv.z, d2);
        d2 = fmaf(sq[D + 4 * c + 3], kv.w, d2);
      }
      s1 = d1 * scale;
      s2 = d2 * scale;
    }
    float c1 = s1, c2 = s2;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      c1 = fmaxf(c1, __shfl_xor_sync(0xffffffffu, c1, off));
      c2 = fmaxf(c2, __shfl_xor_sync(0xffffffffu, c2, off));
    }
    const float n1 = fmaxf(m1, c1), n2 = fmaxf(m2, c2);  // finite: key j0 is visible
    const float a1 = expf(m1 - n1), a2 = expf(m2 - n2);
    const float p1 = (j < n_keys) ? expf(s1 - n1) : 0.f;
    const float p2 = (j < n_keys) ? expf(s2 - n2) : 0.f;
    float t1 = p1, t2 = p2;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      t1 += __shfl_xor_sync(0xffffffffu, t1, off);
      t2 += __shfl_xor_sync(0xffffffffu, t2, off);
    }
    l1 = l1 * a1 + t1;
    l2 = l2 * a2 + t2;
    m1 = n1;
    m2 = n2;
#pragma unroll
    for (int u = 0; u < U; ++u) {
      acc1[u] *= a1;
      acc2[u] *= a2;
    }
    const int nj = min(32, n_keys - j0);
    for (int jj = 0; jj < nj; ++jj) {
      const float w1 = __shfl_sync(0xffffffffu, p1, jj);
      const float w2 = __shfl_sync(0xffffffffu, p2, jj);
      const float* vr = vbase + static_cast<size_t>(j0 + jj) * row_stride;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const float vv = __ldg(vr + lane + 32 * u);
        acc1[u] = fmaf(w1, vv, acc1[u]);
        acc2[u] = fmaf(w2, vv, acc2[u]);
      }
    }
  }
  const float i1 = (l1 > 0.f) ? 1.f / l1 : 0.f;
  const float i2 = (l2 > 0.f) ? 1.f / l2 : 0.f;
#pragma unroll
  for (int u = 0; u < U; ++u) out[lane + 32 * u] = acc1[u] * i1 - lam * (acc2[u] * i2);
  __syncwarp();
}

constexpr int kWarps = 4;

template <int D>
__global__ void __launch_bounds__(32 * kWarps)
prefill_f32_kernel(const float* __restrict__ q, const float* __restrict__ k, const float* __restrict__ v,
                   const float* __restrict__ lambda, float* __restrict__ out, int B, int S, int Hq, int Hkv,
                   int causal) {
  __shared__ float sq[kWarps][2 * D];
  const int warp = threadIdx.x >> 5;
  const int i = blockIdx.x * kWarps + warp;
  const int n_pairs = Hq >> 1;
  const int b = blockIdx.y / n_pairs;
  const int pair = blockIdx.y % n_pairs;
  if (i >= S) return;
  const int g = (2 * pair) / (Hq / Hkv);
  const float* q1 = q + ((static_cast<size_t>(b) * S + i) * Hq + 2 * pair) * D;
  const size_t kv0 = (static_cast<size_t>(b) * S * Hkv + g) * D;
  const size_t orow = (static_cast<size_t>(b) * S + i) * n_pairs + pair;
  const int n_keys = causal ? i + 1 : S;
  diff_row_f32<D>(q1, q1 + D, k + kv0, v + kv0, Hkv * D, n_keys, __ldg(lambda + orow), out + orow * D, sq[warp]);
}

template <int D>
__global__ void __launch_bounds__(32 * kWarps)
decode_f32_kernel(const float* __restrict__ q, const float* __restrict__ kc, const float* __restrict__ vc,
                  const int32_t* __restrict__ seqlens, const float* __restrict__ lambda, float* __restrict__ out,
                  int B, int Smax, int Hq, int Hkv) {
  __shared__ float sq[kWarps][2 * D];
  const int warp = threadIdx.x >> 5;
  const int n_pairs = Hq >> 1;
  const int w = blockIdx.x * kWarps + warp;
  if (w >= B * n_pairs) return;
  const int b = w / n_pairs;
  const int pair = w % n_pairs;
  const int g = (2 * pair) / (Hq / Hkv);
  const int n_keys = min(max(__ldg(seqlens + b), 0), Smax);
  const float* q1 = q + (static_cast<size_t>(b) * Hq + 2 * pair) * D;
  const size_t kv0 = (static_cast<size_t>(b) * Smax * Hkv + g) * D;
  diff_row_f32<D>(q1, q1 + D, kc + kv0, vc + kv0, Hkv * D, n_keys, __ldg(lambda + w), out + static_cast<size_t>(w) * D,
                  sq[warp]);
}

}  // namespace simt

cudaError_t launch_prefill_f32(const float* q, const float* k, const float* v, const float* lambda, float* out,
                               int B, int S, int Hq, int Hkv, int D, int causal, cudaStream_t stream) {
  dim3 grid((S + simt::kWarps - 1) / simt::kWarps, B * (Hq / 2));
  if (D == 64)
    simt::prefill_f32_kernel<64><<<grid, 32 * simt::kWarps, 0, stream>>>(q, k, v, lambda, out, B, S, Hq, Hkv, causal);
  else
    simt::prefill_f32_kernel<128><<<grid, 32 * simt::kWarps, 0, stream>>>(q, k, v, lambda, out, B, S, Hq, Hkv, causal);
  return cudaGetLastError();
}

cudaError_t launch_decode_f32(const float* q, const float* kc, const float* vc, const int32_t* seqlens,
                              const float* lambda, float* out, int B, int Smax, int Hq, int Hkv, int D,
                              cudaStream_t stream) {
  const int warps = B * (Hq / 2);
  dim3 grid((warps + simt::kWarps - 1) / simt::kWarps);
  if (D == 64)
    simt::decode_f32_kernel<64><<<grid, 32 * simt::kWarps, 0, stream>>>(q, kc, vc, seqlens, lambda, out, B, Smax, Hq, Hkv);
  else
    simt::decode_f32_kernel<128><<<grid, 32 * simt::kWarps, 0, stream>>>(q, kc, vc, seqlens, lambda, out, B, Smax, Hq, Hkv);
  return cudaGetLastError();
}

}  // namespace da2
