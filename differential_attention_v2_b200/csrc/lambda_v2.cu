// lambda_v2.cu -- the V2 lambda projection: lambda[t, p] = sigmoid(x[t] . W[:, p] + bias[p]).
//
// "Differential Transformer V2 soll KI-Training stabiler machen", section "Weniger
// Ausreisser und Gradientenspitzen": V2 drops V1's per-head normalisation and instead
// projects, for every token and every head, a lambda bounded by a sigmoid. Here "head" is
// the output head, i.e. the pair, and the projection input is the token's hidden state x.
//
// x [T, d_model] bf16 and W [d_model, n_pairs] bf16 give a skinny GEMM (n_pairs <= 64) whose
// cost is reading x once from HBM. Each CTA also reads all of W (d_model x n_pairs, 256 KB at
// d_model = 4096 and 32 pairs) from L2 for every tile of tokens it computes, so the token tile
// must be large for W's share of the shared-memory fill to stay small: with 32-token tiles W
// doubled the bytes per stage and the kernel read x at half of HBM bandwidth. The host sizes
// the tile so that about one tile lands on every SM: 16 x nw tokens with nw = ceil(T / (16 x
// SMs)) warps, at most 8 (T = 16384 on 148 SMs: 7 warps, 112 tokens, 147 CTAs); larger T
// loops over 128-token tiles. Warp w computes tokens 16w .. 16w+15 of the tile and all pairs
// on mma.sync m16n8k16 (bf16 in, fp32 accumulate); x and W chunks of 64 along d_model stream
// through a 6-stage ring filled by cp.async (up to 150 KB, one CTA per SM). The epilogue adds
// the bias and applies the sigmoid with the accurate expf, writing fp32 lambda [T, n_pairs]
// -- the layout of the prefill ([B*S, Hq/2]) and decode ([B, Hq/2]) lambda arguments.

#include "internal.h"
#include "ptx.cuh"

namespace da2 {
namespace lambda2 {

constexpr int kMaxWarps = 8;            // a tile is 16 tokens per warp
constexpr int kMaxTok = 16 * kMaxWarps;
constexpr int kChunk = 64;   // d_model per stage
constexpr int kStages = 6;   // ring depth

template <int NT>
constexpr int smem_bytes() { return kStages * (kMaxTok * kChunk * 2 + kChunk * (NT + 1) * 16); }

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// NT: 8-pair column tiles, padded to an even count (pairs past n_pairs read zeros). The block
// has nw = blockDim.x / 32 warps and its tiles hold 16 nw tokens.
template <int NT>
__global__ void __launch_bounds__(32 * kMaxWarps, 1)
lambda_v2_kernel(const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ w,
                 const float* __restrict__ bias, float* __restrict__ out, int T, int d_model, int n_pairs) {
  constexpr int kWChunks = NT + 1;                     // 16-byte chunks per W row (+1 padding)
  constexpr uint32_t kXBytes = kMaxTok * kChunk * 2;   // x stage (16 KB: room for 128 tokens)
  constexpr uint32_t kWBytes = kChunk * kWChunks * 16; // W stage
  extern __shared__ __align__(128) uint8_t smem[];
  const uint32_t sx = smem_u32(smem);
  const uint32_t sw = sx + kStages * kXBytes;

  const int n_threads = blockDim.x;
  const int tile_tok = 16 * (n_threads >> 5);
  const int n_tiles = (T + tile_tok - 1) / tile_tok;
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int n_chunks = d_model / kChunk;
  const int a_row = 16 * warp + (lane & 7) + ((lane >> 3) & 1) * 8;  // x: (r0,k0)(r8,k0)(r0,k8)(r8,k8)
  const int a_csel = (lane >> 4) & 1;
  const int b_krow = (lane & 7) + (lane >> 3 & 1) * 8;                 // W: (k0,n0)(k8,n0)(k0,n8)(k8,n8)
  const int b_nsel = (lane >> 4) & 1;

  for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
    const int tok0 = tile * tile_tok;
    // x tile: row r (token), 16-byte chunk c of the 64-wide slice, stored at chunk c ^ (r & 7)
    auto load_stage = [&](int st, int kc) {
      for (int idx = tid; idx < tile_tok * 8; idx += n_threads) {
        const int r = idx >> 3, c = idx & 7;
        const int t = tok0 + r;
        const __nv_bfloat16* src = x + static_cast<size_t>(t < T ? t : 0) * d_model + kc * kChunk + c * 8;
        cp_async16(sx + st * kXBytes + r * 128 + ((c ^ (r & 7)) << 4), src, t < T ? 16 : 0);
      }
      // W slice: row k of the chunk, chunk c = pairs 8c .. 8c+7
      for (int idx = tid; idx < kChunk * NT; idx += n_threads) {
        const int k = idx / NT, c = idx % NT;
        const bool valid = 8 * c < n_pairs;
        const __nv_bfloat16* src = w + static_cast<size_t>(kc * kChunk + k) * n_pairs + (valid ? 8 * c : 0);
        cp_async16(sw + st * kWBytes + (k * kWChunks + c) * 16, src, valid ? 16 : 0);
      }
      cp_async_commit();
    };

    float acc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;

    // one commit group per chunk (empty groups past the end keep the count uniform)
#pragma unroll
    for (int s = 0; s < kStages - 1; ++s) {
      if (s < n_chunks) load_stage(s, s);
      else cp_async_commit();
    }
    for (int kc = 0; kc < n_chunks; ++kc) {
      const int st = kc % kStages;
      cp_async_wait<kStages - 2>();  // chunk kc has landed (this thread's copies)
      __syncthreads();               // ... everyone's; and chunk kc-1's stage is free
      if (kc + kStages - 1 < n_chunks) load_stage((kc + kStages - 1) % kStages, kc + kStages - 1);
      else cp_async_commit();
#pragma unroll
      for (int ks = 0; ks < kChunk / 16; ++ks) {
        const int chunk = 2 * ks + a_csel;
        uint32_t a0, a1, a2, a3;
        ldmatrix_x4(sx + st * kXBytes + a_row * 128 + ((chunk ^ (a_row & 7)) << 4), a0, a1, a2, a3);
#pragma unroll
        for (int np = 0; np < NT / 2; ++np) {
          uint32_t b0, b1, b2, b3;
          const int krow = 16 * ks + b_krow;
          ldmatrix_x4_trans(sw + st * kWBytes + (krow * kWChunks + 2 * np + b_nsel) * 16, b0, b1, b2, b3);
          mma_m16n8k16_bf16(acc[2 * np], a0, a1, a2, a3, b0, b1);
          mma_m16n8k16_bf16(acc[2 * np + 1], a0, a1, a2, a3, b2, b3);
        }
      }
    }
    // every copy of this tile has landed and every warp has left its loop before the next
    // tile's prologue refills the ring
    cp_async_wait<0>();
    __syncthreads();

    const int gl = lane >> 2, tq = lane & 3;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int pcol = 8 * nt + 2 * tq;
      if (pcol >= n_pairs) continue;
      const float b0 = bias ? __ldg(bias + pcol) : 0.f;
      const float b1 = bias ? __ldg(bias + pcol + 1) : 0.f;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int t = tok0 + 16 * warp + gl + 8 * h;
        if (t >= T) continue;
        const float z0 = acc[nt][2 * h] + b0;
        const float z1 = acc[nt][2 * h + 1] + b1;
        float2 v;
        v.x = 1.f / (1.f + expf(-z0));
        v.y = 1.f / (1.f + expf(-z1));
        *reinterpret_cast<float2*>(out + static_cast<size_t>(t) * n_pairs + pcol) = v;
      }
    }
  }
}

}  // namespace lambda2

cudaError_t launch_lambda_v2(const __nv_bfloat16* x, const __nv_bfloat16* w, const float* bias, int T, int d_model,
                             int n_pairs, float* out, cudaStream_t stream) {
  using namespace lambda2;
  int device = 0, n_sms = 0;
  cudaError_t e = cudaGetDevice(&device);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&n_sms, cudaDevAttrMultiProcessorCount, device);
  if (e != cudaSuccess) return e;
  // about one tile per SM: nw warps (16 tokens each) with 16 nw * n_sms >= T, at most 8
  const int per_sm = (T + n_sms - 1) / n_sms;
  const int nw = per_sm <= 16 ? 1 : (per_sm + 15) / 16 > kMaxWarps ? kMaxWarps : (per_sm + 15) / 16;
  const int tile = 16 * nw;
  const int n_tiles = (T + tile - 1) / tile;
  const dim3 grid(n_tiles < n_sms ? n_tiles : n_sms);
  const int nt = (n_pairs + 15) / 16 * 2;  // 8-pair tiles, even
  auto run = [&](auto kernel, int smem) {
    cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err != cudaSuccess) return err;
    kernel<<<grid, 32 * nw, smem, stream>>>(x, w, bias, out, T, d_model, n_pairs);
    return cudaGetLastError();
  };
  switch (nt) {
    case 2: return run(lambda_v2_kernel<2>, smem_bytes<2>());
    case 4: return run(lambda_v2_kernel<4>, smem_bytes<4>());
    case 6: return run(lambda_v2_kernel<6>, smem_bytes<6>());
    case 8: return run(lambda_v2_kernel<8>, smem_bytes<8>());
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace da2
