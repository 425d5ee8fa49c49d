// lambda_v2.cu -- the V2 lambda projection: lambda[t, p] = sigmoid(x[t] . W[:, p] + bias[p]).
//
// "Differential Transformer V2 soll KI-Training stabiler machen", section "Weniger
// Ausreisser und Gradientenspitzen": V2 drops V1's per-head normalisation and instead
// projects, for every token and every head, a lambda bounded by a sigmoid. Here "head" is
// the output head, i.e. the pair, and the projection input is the token's hidden state x.
//
// x [T, d_model] bf16 and W [d_model, n_pairs] bf16 give a skinny GEMM (n_pairs <= 64) whose
// cost should be reading x once from HBM: 32 FLOP per byte of x at 32 pairs, more than the
// legacy warp-level MMA path sustains (it held an earlier kernel of this projection to half
// of HBM bandwidth, about 4 us per 16k tokens for every 8 pairs). Here the product runs on
// the 5th-generation tensor cores:
//
//   * one CTA per 128-token tile: D[128 tokens x 64] = x_tile[128 x d_model] W[d_model x 64]
//     on tcgen05.mma (M = 128, N = 64, K = 16), fp32 accumulators in 64 TMEM columns;
//   * two producer warps stream 128-wide chunks of d_model by TMA, each through its own
//     4-stage ring: the x tile (128 rows x 128 as two 64-wide boxes, K-major, 128-byte
//     swizzle, the A operand) and the W chunk (128 rows of d_model x 64 pair columns as two
//     64-row boxes, MN-major, the B operand; the tensor map covers n_pairs columns, so the
//     columns past n_pairs read as zeros). What bounds it is the shape of the x stream: short
//     pieces of 128 rows 8 KB apart (a probe of the access pattern alone, no compute, read
//     128-byte pieces at 5.0 TB/s against 5.8 for contiguous 4 KB pieces). Measured on B200
//     (16k tokens x 4096, 32 pairs, same box, alternating rounds): 256-byte pieces in 4 + 4
//     stages 4.43 TB/s against 4.16 for 128-byte pieces in 6 + 6 stages; 512-byte pieces fit
//     only 2 + 2 stages (4.18). Earlier, with 128-byte pieces: deeper x rings with shallower
//     W rings were slower (10 + 3: 3.82, 12 + 2: 3.19), and so was starting each CTA's walk
//     over d_model at its own chunk (3.92);
//   * an MMA warp issues the eight K-steps of each chunk and releases the stage by a commit;
//   * four epilogue warps (one per TMEM lane quarter) read their rows' accumulators, add the
//     bias, apply the sigmoid with the accurate expf and write fp32 lambda [T, n_pairs] -- the
//     layout of the prefill ([B*S, Hq/2]) and decode ([B, Hq/2]) lambda arguments.
//
// Every wait is bounded; on expiry the kernel records kErrLambdaWait and returns.

#include "bounds.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace da2 {
namespace lambda2 {

constexpr int BM = 128;                            // tokens per tile (MMA M)
constexpr int kBoxes = 2;                          // 64-wide TMA boxes per stage
constexpr int BK = 64 * kBoxes;                    // d_model per stage
constexpr int BN = 64;                             // W columns per stage (MMA N)
constexpr int kXStages = 4;
constexpr int kWStages = 4;
constexpr int kThreads = 224;                      // x producer, MMA issuer, 4 epilogue warps, W producer
constexpr uint32_t kXBox = BM * 64 * 2;            // 16 KB: 128 rows x 64 of d_model
constexpr uint32_t kWBox = 64 * BN * 2;            // 8 KB: 64 rows of d_model x 64 columns
constexpr uint32_t kXBytes = kBoxes * kXBox;
constexpr uint32_t kWBytes = kBoxes * kWBox;
constexpr uint32_t kOffW = kXStages * kXBytes;
constexpr uint32_t kOffBar = kOffW + kWStages * kWBytes;
constexpr int kNumBars = 2 * kXStages + 2 * kWStages + 1;
constexpr uint32_t kOffMisc = kOffBar + 8 * kNumBars;
constexpr uint32_t kSmemBytes = kOffMisc + 16 + 1024;  // + slack for 1024-B alignment
constexpr uint32_t kTmemCols = 64;
__global__ void __launch_bounds__(kThreads, 1)
lambda_v2_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                 const float* __restrict__ bias, float* __restrict__ out, int* err, int T, int d_model,
                 int n_pairs) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  auto xfull = [&](int s) -> uint32_t { return sbase + kOffBar + 8u * s; };
  auto xempty = [&](int s) -> uint32_t { return sbase + kOffBar + 8u * (kXStages + s); };
  auto wfull = [&](int s) -> uint32_t { return sbase + kOffBar + 8u * (2 * kXStages + s); };
  auto wempty = [&](int s) -> uint32_t { return sbase + kOffBar + 8u * (2 * kXStages + kWStages + s); };
  const uint32_t dfull = sbase + kOffBar + 8u * (kNumBars - 1);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 8);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int tok0 = blockIdx.x * BM;
  // d_model is a multiple of 64: a last chunk of 64 reads its second box past the end of x
  // and W, which the copies fill with zeros (products that add nothing)
  const int n_chunks = (d_model + BK - 1) / BK;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kNumBars; ++i) mbar_init(sbase + kOffBar + 8u * i, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmW);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 || warp == 6) {
    // ------------------------------------------------- TMA producers: x (warp 0), W (warp 6)
    if (lane == 0) {
      const bool is_x = warp == 0;
      const int stages = is_x ? kXStages : kWStages;
      int issued = 0;
      for (int kc = 0; kc < n_chunks; ++kc) {
        const int s = kc % stages;
        const int c = kc;  // chunk of d_model
        const uint32_t fb = is_x ? xfull(s) : wfull(s);
        if (!mbar_wait(is_x ? xempty(s) : wempty(s), ((kc / stages) & 1) ^ 1, abort_flag)) break;
        mbar_arrive_expect_tx(fb, is_x ? kXBytes : kWBytes);
        if (!checked(c * BK < d_model, err)) continue;
        for (int b = 0; b < kBoxes; ++b) {
          if (is_x)
            tma_load_2d(sbase + s * kXBytes + b * kXBox, &tmX, fb, c * BK + 64 * b, tok0);
          else
            tma_load_2d(sbase + kOffW + s * kWBytes + b * kWBox, &tmW, fb, 0, c * BK + 64 * b);
        }
        issued = kc + 1;
      }
      if (*abort_flag) {
        // every issued copy lands before the shared memory is released; each wait has its own limit
        for (int kc = issued - stages > 0 ? issued - stages : 0; kc < issued; ++kc) {
          volatile int na = 0;
          mbar_wait(is_x ? xfull(kc % stages) : wfull(kc % stages), (kc / stages) & 1, &na);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(BM, BN, true);
      bool ok = checked((tmem & 0xFFFFu) == 0u, err);
      for (int kc = 0; ok && kc < n_chunks; ++kc) {
        const int s = kc % kXStages, sw = kc % kWStages;
        if (!(ok = mbar_wait(xfull(s), (kc / kXStages) & 1, abort_flag))) break;
        if (!(ok = mbar_wait(wfull(sw), (kc / kWStages) & 1, abort_flag))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk) {
          // A: x rows, K-major, K-step kk in box kk / 4 at +32 bytes per step of the 128-byte
          // swizzled row; B: W rows of d_model (16 per K-step, 2 KB apart, the boxes back to
          // back), the 64 columns contiguous
          const uint64_t adesc = sdesc_sw128(sbase + s * kXBytes + (kk >> 2) * kXBox + (kk & 3) * 32, 16, 1024);
          const uint64_t bdesc = sdesc_sw128(sbase + kOffW + sw * kWBytes + kk * 2048, kWBox, 1024);
          mma_bf16_ss(tmem, adesc, bdesc, idesc, (kc > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(xempty(s));
        tc_commit(wempty(sw));
      }
      tc_commit(dfull);  // also the drain: every MMA of the tile is complete when it fires
      volatile int na = 0;
      mbar_wait(dfull, 0, &na);
    }
  } else {
    // ------------------------------------------------------------------ epilogue
    // warps 2-5; warp w reads TMEM lanes 32 (w % 4) .. +31: rows of the tile
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;
    const int t = tok0 + r;
    const bool ok = __all_sync(0xffffffffu, mbar_wait(dfull, 0, abort_flag));
    if (ok) {
      tc_fence_after();
      const uint32_t trow = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 32) {
        if (c0 >= n_pairs) break;  // uniform: n_pairs is the same for every thread
        uint32_t a[32];
        tmem_ld_32x32b_x32(trow + c0, a);
        tmem_ld_wait(a);
        if (t < T) {
          float* dst = out + static_cast<size_t>(t) * n_pairs + c0;
          const int nc = n_pairs - c0 < 32 ? n_pairs - c0 : 32;  // a multiple of 8
#pragma unroll
          for (int v = 0; v < 32; v += 4) {
            if (v >= nc) break;
            float4 o;
            float* po = &o.x;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float z = __uint_as_float(a[v + e]) + (bias ? __ldg(bias + c0 + v + e) : 0.f);
              po[e] = 1.f / (1.f + expf(-z));
            }
            *reinterpret_cast<float4*>(dst + v) = o;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag) atomicCAS(err, 0, kErrLambdaWait);
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace lambda2

cudaError_t launch_lambda_v2(const CUtensorMap& tmX, const CUtensorMap& tmW, const float* bias, int T, int d_model,
                             int n_pairs, float* out, int* err, cudaStream_t stream) {
  using namespace lambda2;
  cudaError_t e = cudaFuncSetAttribute(lambda_v2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  const dim3 grid((T + BM - 1) / BM);
  lambda_v2_kernel<<<grid, kThreads, kSmemBytes, stream>>>(tmX, tmW, bias, out, err, T, d_model, n_pairs);
  return cudaGetLastError();
}

}  // namespace da2
