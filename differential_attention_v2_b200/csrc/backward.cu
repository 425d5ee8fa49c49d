// backward.cu -- gradients of the bf16 DiffAttn V2 prefill (training).
//
// Forward (per pair p of heads h1 = 2p, h2 = 2p+1 over KV head g; "Differential Attention
// (V2)" lesson, "The differential concept"; causal mask of the "Attention variants" lesson):
//   A_b = softmax(Q_b K^T / sqrt(D)),   O_b = A_b V,   out = O_1 - lambda * O_2.
// Chain rule, with c_1 = 1 and c_2 = -lambda (per query row), dO the upstream gradient:
//   dlambda   = -dO . O_2
//   dV       += sum_b (c_b A_b)^T dO
//   dP_b      = dO V^T,   E_b = dO . O_b   (per row)
//   dS_b      = c_b * A_b (.) (dP_b - E_b)             (softmax backward, E_b = rowsum(A_b dP_b))
//   dQ_b      = dS_b K / sqrt(D),   dK += sum_b dS_b^T Q_b / sqrt(D)
// A_b is recomputed from the forward's per-row log-sum-exp: A_b = 2^(s log2(e)/sqrt(D) - lse_b).
//
// Three kernels, FlashAttention-2 style, on the warp-level tensor cores (mma.sync m16n8k16,
// bf16 operands, fp32 accumulation); no atomics, results are deterministic:
//   * preprocess: E_b and dlambda, one warp per (token, pair);
//   * dK/dV: a CTA owns 64 keys of one KV head and loops over every query head of its GQA
//     group and every query tile that sees the keys; four warps own 16 keys each;
//   * dQ: a CTA owns 64 query rows of one head and loops over the key tiles they see.
// Shared-memory tiles are rows of 128 bf16 (256 B) with the 16-byte chunks XOR-swizzled by
// the row index, so ldmatrix reads are free of bank conflicts.

#include "internal.h"
#include "ptx.cuh"

namespace da2 {
namespace bwd {

constexpr int HD = 128;

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

// byte offset of 16-byte chunk c (0..15) of row r in a swizzled [rows][128 bf16] tile
__device__ __forceinline__ uint32_t sw(int r, int c) { return static_cast<uint32_t>(r * 256 + ((c ^ (r & 7)) << 4)); }

// Copy `rows` rows of 128 bf16 (global row stride `stride` elements) into a swizzled tile;
// rows at or past `valid` read zeros.
__device__ __forceinline__ void load_tile(uint32_t dst, const __nv_bfloat16* src, size_t stride, int rows, int valid,
                                          int tid, int nthreads) {
  for (int i = tid; i < rows * 16; i += nthreads) {
    const int r = i >> 4, c = i & 15;
    const bool ok = r < valid;
    cp_async16(dst + sw(r, c), src + (ok ? static_cast<size_t>(r) * stride : 0) + c * 8, ok ? 16 : 0);
  }
}

// ------------------------------------------------------------------------ preprocess
// E[row, h] = dO[row, p] . O_branch[row, h] for both heads of pair p; dlambda = -E[row, 2p+1].
__global__ void __launch_bounds__(128)
preprocess_kernel(const __nv_bfloat16* __restrict__ dout, const __nv_bfloat16* __restrict__ o_branch,
                  float* __restrict__ E, float* __restrict__ dlam, long long rows, int n_pairs) {
  const long long w = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (w >= rows * n_pairs) return;
  const long long row = w / n_pairs;
  const int p = static_cast<int>(w % n_pairs);
  const uint2 g = __ldg(reinterpret_cast<const uint2*>(dout + w * HD) + lane);
  float e[2];
#pragma unroll
  for (int br = 0; br < 2; ++br) {
    const uint2 o = __ldg(reinterpret_cast<const uint2*>(o_branch + (row * (2 * n_pairs) + 2 * p + br) * HD) + lane);
    const float2 g0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&g.x));
    const float2 g1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&g.y));
    const float2 o0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&o.x));
    const float2 o1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&o.y));
    float v = g0.x * o0.x + g0.y * o0.y + g1.x * o1.x + g1.y * o1.y;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    e[br] = v;
  }
  if (lane == 0) {
    E[row * (2 * n_pairs) + 2 * p] = e[0];
    E[row * (2 * n_pairs) + 2 * p + 1] = e[1];
    dlam[w] = -e[1];
  }
}

struct Params {
  const __nv_bfloat16 *q, *k, *v, *dout;  // [B,S,Hq,D], [B,S,Hkv,D] x2, [B,S,Hq/2,D]
  const float *lambda, *lse, *E;          // [B,S,Hq/2], [B,S,Hq], [B,S,Hq]
  __nv_bfloat16 *dq, *dk, *dv;            // [B,S,Hq,D], [B,S,Hkv,D] x2
  int B, S, Hq, Hkv, causal;
  float scale, scale_log2;                // 1/sqrt(D), log2(e)/sqrt(D)
};

// --------------------------------------------------------------------------- dK / dV
constexpr int kKvRows = 64;  // keys per CTA (16 per warp)
constexpr int kQRows = 32;   // query rows per inner step

// K, V tiles; Q_1, Q_2, dO tiles of the step; per-row lse_1, lse_2, E_1, E_2, lambda
constexpr int kDkdvSmem = 2 * kKvRows * 256 + 3 * kQRows * 256 + 5 * kQRows * 4;

// A CTA owns 64 keys of KV head g and walks the pairs of g's group: per step of 32 query
// rows it forms S_1^T, S_2^T (recomputed), dP^T = V dO^T (shared by both branches), the
// combined weights W^T = P_1^T - lambda P_2^T in fp32 (one bf16 rounding, so W stays accurate
// where the branches cancel), dS_b^T = c_b P_b^T (dP^T - E_b), then dV += W^T dO and
// dK += dS_1^T Q_1 + dS_2^T Q_2.
__global__ void __launch_bounds__(128)
dkdv_kernel(const Params p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sK = smem_u32(smem), sV = sK + kKvRows * 256;
  const uint32_t sQ1 = sV + kKvRows * 256, sQ2 = sQ1 + kQRows * 256, sO = sQ2 + kQRows * 256;
  float* s_lse1 = reinterpret_cast<float*>(smem + 2 * kKvRows * 256 + 3 * kQRows * 256);
  float* s_lse2 = s_lse1 + kQRows;
  float* s_E1 = s_lse2 + kQRows;
  float* s_E2 = s_E1 + kQRows;
  float* s_lam = s_E2 + kQRows;

  const int tile = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gl = lane >> 2, tq = lane & 3;
  const int k0 = tile * kKvRows;
  const int group = p.Hq / p.Hkv, n_pairs = p.Hq >> 1;
  const size_t kv_stride = static_cast<size_t>(p.Hkv) * HD;

  load_tile(sK, p.k + (static_cast<size_t>(b) * p.S + k0) * kv_stride + g * HD, kv_stride, kKvRows, p.S - k0, tid, 128);
  load_tile(sV, p.v + (static_cast<size_t>(b) * p.S + k0) * kv_stride + g * HD, kv_stride, kKvRows, p.S - k0, tid, 128);

  float dv[16][4], dk[16][4];
#pragma unroll
  for (int n = 0; n < 16; ++n) dv[n][0] = dv[n][1] = dv[n][2] = dv[n][3] = dk[n][0] = dk[n][1] = dk[n][2] = dk[n][3] = 0.f;

  // A fragments of this warp's 16 keys come from the K / V tiles
  const int a_row = 16 * warp + (lane & 7) + ((lane >> 3) & 1) * 8;
  const int a_csel = (lane >> 4) & 1;
  const int key_a = k0 + 16 * warp + gl, key_b = key_a + 8;

  for (int pr = 0; pr < group / 2; ++pr) {
    const int pair = g * (group / 2) + pr, h1 = 2 * pair;
    const int q_first = p.causal ? (k0 / kQRows) * kQRows : 0;
    for (int qt = q_first; qt < p.S; qt += kQRows) {
      __syncthreads();  // the previous step's tiles are no longer read
      const size_t qrow0 = static_cast<size_t>(b) * p.S + qt;
      const size_t q_stride = static_cast<size_t>(p.Hq) * HD;
      load_tile(sQ1, p.q + qrow0 * q_stride + h1 * HD, q_stride, kQRows, p.S - qt, tid, 128);
      load_tile(sQ2, p.q + qrow0 * q_stride + (h1 + 1) * HD, q_stride, kQRows, p.S - qt, tid, 128);
      load_tile(sO, p.dout + qrow0 * n_pairs * HD + pair * HD, static_cast<size_t>(n_pairs) * HD, kQRows, p.S - qt,
                tid, 128);
      if (tid < kQRows) {
        const bool ok = qt + tid < p.S;
        const size_t r = qrow0 + (ok ? tid : 0);
        s_lse1[tid] = ok ? __ldg(p.lse + r * p.Hq + h1) : 0.f;
        s_lse2[tid] = ok ? __ldg(p.lse + r * p.Hq + h1 + 1) : 0.f;
        s_E1[tid] = ok ? __ldg(p.E + r * p.Hq + h1) : 0.f;
        s_E2[tid] = ok ? __ldg(p.E + r * p.Hq + h1 + 1) : 0.f;
        s_lam[tid] = ok ? __ldg(p.lambda + r * n_pairs + pair) : 0.f;
      }
      cp_async_wait_all();
      __syncthreads();

      // S_b^T = K_w Q_b^T and dP^T = V_w dO^T: 16 keys x 32 queries, K = d
      float s1[4][4], s2[4][4], dp[4][4];
#pragma unroll
      for (int n = 0; n < 4; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) s1[n][e] = s2[n][e] = dp[n][e] = 0.f;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        uint32_t ka0, ka1, ka2, ka3, va0, va1, va2, va3;
        ldmatrix_x4(sK + sw(a_row, 2 * kk + a_csel), ka0, ka1, ka2, ka3);
        ldmatrix_x4(sV + sw(a_row, 2 * kk + a_csel), va0, va1, va2, va3);
#pragma unroll
        for (int np = 0; np < 2; ++np) {
          // B fragments: rows = queries of n-tiles 2np, 2np+1; chunks 2kk, 2kk+1 of d
          const int brow = 16 * np + ((lane >> 4) & 1) * 8 + (lane & 7);
          const int bc = 2 * kk + ((lane >> 3) & 1);
          uint32_t b0, b1, b2, b3;
          ldmatrix_x4(sQ1 + sw(brow, bc), b0, b1, b2, b3);
          mma_m16n8k16_bf16(s1[2 * np], ka0, ka1, ka2, ka3, b0, b1);
          mma_m16n8k16_bf16(s1[2 * np + 1], ka0, ka1, ka2, ka3, b2, b3);
          ldmatrix_x4(sQ2 + sw(brow, bc), b0, b1, b2, b3);
          mma_m16n8k16_bf16(s2[2 * np], ka0, ka1, ka2, ka3, b0, b1);
          mma_m16n8k16_bf16(s2[2 * np + 1], ka0, ka1, ka2, ka3, b2, b3);
          ldmatrix_x4(sO + sw(brow, bc), b0, b1, b2, b3);
          mma_m16n8k16_bf16(dp[2 * np], va0, va1, va2, va3, b0, b1);
          mma_m16n8k16_bf16(dp[2 * np + 1], va0, va1, va2, va3, b2, b3);
        }
      }
      // W^T, dS_1^T, dS_2^T as A fragments of the two 16-query k-steps; columns are queries
      uint32_t wa[2][4], d1a[2][4], d2a[2][4];
#pragma unroll
      for (int n = 0; n < 4; ++n) {
        float w[4], d1[4], d2[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int col = 8 * n + 2 * tq + (e & 1);
          const int qi = qt + col;
          const int key = (e < 2) ? key_a : key_b;
          const bool vis = qi < p.S && key < p.S && (!p.causal || key <= qi);
          const float p1 = vis ? fast_exp2(s1[n][e] * p.scale_log2 - s_lse1[col]) : 0.f;
          const float p2 = vis ? fast_exp2(s2[n][e] * p.scale_log2 - s_lse2[col]) : 0.f;
          const float lam = s_lam[col];
          w[e] = __fmaf_rn(-lam, p2, p1);
          d1[e] = p1 * (dp[n][e] - s_E1[col]);
          d2[e] = -lam * p2 * (dp[n][e] - s_E2[col]);
        }
        const int ks = n >> 1, hi = n & 1;
        wa[ks][2 * hi + 0] = pack_bf16x2(w[0], w[1]);
        wa[ks][2 * hi + 1] = pack_bf16x2(w[2], w[3]);
        d1a[ks][2 * hi + 0] = pack_bf16x2(d1[0], d1[1]);
        d1a[ks][2 * hi + 1] = pack_bf16x2(d1[2], d1[3]);
        d2a[ks][2 * hi + 0] = pack_bf16x2(d2[0], d2[1]);
        d2a[ks][2 * hi + 1] = pack_bf16x2(d2[2], d2[3]);
      }
      // dV += W^T dO and dK += dS_1^T Q_1 + dS_2^T Q_2: 16 keys x 128 d, K = 32 queries
#pragma unroll
      for (int ks = 0; ks < 2; ++ks) {
#pragma unroll
        for (int np = 0; np < 8; ++np) {
          // B fragments from rows = queries 16ks .. 16ks+15, chunks 2np, 2np+1 of d (transposed)
          const int brow = 16 * ks + ((lane >> 3) & 1) * 8 + (lane & 7);
          const int bc = 2 * np + ((lane >> 4) & 1);
          uint32_t b0, b1, b2, b3;
          ldmatrix_x4_trans(sO + sw(brow, bc), b0, b1, b2, b3);
          mma_m16n8k16_bf16(dv[2 * np], wa[ks][0], wa[ks][1], wa[ks][2], wa[ks][3], b0, b1);
          mma_m16n8k16_bf16(dv[2 * np + 1], wa[ks][0], wa[ks][1], wa[ks][2], wa[ks][3], b2, b3);
          ldmatrix_x4_trans(sQ1 + sw(brow, bc), b0, b1, b2, b3);
          mma_m16n8k16_bf16(dk[2 * np], d1a[ks][0], d1a[ks][1], d1a[ks][2], d1a[ks][3], b0, b1);
          mma_m16n8k16_bf16(dk[2 * np + 1], d1a[ks][0], d1a[ks][1], d1a[ks][2], d1a[ks][3], b2, b3);
          ldmatrix_x4_trans(sQ2 + sw(brow, bc), b0, b1, b2, b3);
          mma_m16n8k16_bf16(dk[2 * np], d2a[ks][0], d2a[ks][1], d2a[ks][2], d2a[ks][3], b0, b1);
          mma_m16n8k16_bf16(dk[2 * np + 1], d2a[ks][0], d2a[ks][1], d2a[ks][2], d2a[ks][3], b2, b3);
        }
      }
    }
  }
  // write dK (scaled by 1/sqrt(D)) and dV for this warp's 16 keys
#pragma unroll
  for (int n = 0; n < 16; ++n) {
#pragma unroll
    for (int hrow = 0; hrow < 2; ++hrow) {
      const int key = hrow ? key_b : key_a;
      if (key >= p.S) continue;
      const size_t off = (static_cast<size_t>(b) * p.S + key) * kv_stride + g * HD + 8 * n + 2 * tq;
      *reinterpret_cast<uint32_t*>(p.dk + off) = pack_bf16x2(dk[n][2 * hrow] * p.scale, dk[n][2 * hrow + 1] * p.scale);
      *reinterpret_cast<uint32_t*>(p.dv + off) = pack_bf16x2(dv[n][2 * hrow], dv[n][2 * hrow + 1]);
    }
  }
}

// --------------------------------------------------------------------------------- dQ
constexpr int kQTile = 64;   // query rows per CTA (16 per warp)
constexpr int kKStep = 32;   // keys per inner step
constexpr int kDqSmem = 2 * kQTile * 256 + 2 * kKStep * 256;

__global__ void __launch_bounds__(128)
dq_kernel(const Params p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sQ = smem_u32(smem), sO = sQ + kQTile * 256;
  const uint32_t sK = sO + kQTile * 256, sV = sK + kKStep * 256;

  const int qtile = blockIdx.x, hq = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gl = lane >> 2, tq = lane & 3;
  const int q0 = qtile * kQTile;
  const int group = p.Hq / p.Hkv, n_pairs = p.Hq >> 1;
  const int g = hq / group, pair = hq >> 1, br = hq & 1;
  const size_t kv_stride = static_cast<size_t>(p.Hkv) * HD;
  const size_t qrow0 = static_cast<size_t>(b) * p.S + q0;

  load_tile(sQ, p.q + qrow0 * p.Hq * HD + hq * HD, static_cast<size_t>(p.Hq) * HD, kQTile, p.S - q0, tid, 128);
  load_tile(sO, p.dout + qrow0 * n_pairs * HD + pair * HD, static_cast<size_t>(n_pairs) * HD, kQTile, p.S - q0, tid,
            128);
  cp_async_wait_all();
  __syncthreads();

  // this warp's 16 query rows as A fragments (kept in registers), and their row statistics
  const int a_row = 16 * warp + (lane & 7) + ((lane >> 3) & 1) * 8;
  const int a_csel = (lane >> 4) & 1;
  uint32_t qa[8][4], oa[8][4];
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    ldmatrix_x4(sQ + sw(a_row, 2 * kk + a_csel), qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3]);
    ldmatrix_x4(sO + sw(a_row, 2 * kk + a_csel), oa[kk][0], oa[kk][1], oa[kk][2], oa[kk][3]);
  }
  const int row_a = q0 + 16 * warp + gl, row_b = row_a + 8;
  float lse[2], E[2], c[2];
#pragma unroll
  for (int hr = 0; hr < 2; ++hr) {
    const int r = hr ? row_b : row_a;
    const bool ok = r < p.S;
    const size_t ri = static_cast<size_t>(b) * p.S + (ok ? r : 0);
    lse[hr] = ok ? __ldg(p.lse + ri * p.Hq + hq) : 0.f;
    E[hr] = ok ? __ldg(p.E + ri * p.Hq + hq) : 0.f;
    c[hr] = br ? (ok ? -__ldg(p.lambda + ri * n_pairs + pair) : 0.f) : 1.f;
  }

  float dq[16][4];
#pragma unroll
  for (int n = 0; n < 16; ++n) dq[n][0] = dq[n][1] = dq[n][2] = dq[n][3] = 0.f;

  const int k_end = p.causal ? min(p.S, q0 + kQTile) : p.S;
  for (int kt = 0; kt < k_end; kt += kKStep) {
    __syncthreads();
    load_tile(sK, p.k + (static_cast<size_t>(b) * p.S + kt) * kv_stride + g * HD, kv_stride, kKStep, p.S - kt, tid, 128);
    load_tile(sV, p.v + (static_cast<size_t>(b) * p.S + kt) * kv_stride + g * HD, kv_stride, kKStep, p.S - kt, tid, 128);
    cp_async_wait_all();
    __syncthreads();

    // S = Q_w K^T and dP = dO_w V^T: 16 rows x 32 keys, K = d
    float s[4][4], dp[4][4];
#pragma unroll
    for (int n = 0; n < 4; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = dp[n][0] = dp[n][1] = dp[n][2] = dp[n][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
#pragma unroll
      for (int np = 0; np < 2; ++np) {
        const int brow = 16 * np + ((lane >> 4) & 1) * 8 + (lane & 7);
        const int bc = 2 * kk + ((lane >> 3) & 1);
        uint32_t k0_, k1_, k2_, k3_, v0, v1, v2, v3;
        ldmatrix_x4(sK + sw(brow, bc), k0_, k1_, k2_, k3_);
        ldmatrix_x4(sV + sw(brow, bc), v0, v1, v2, v3);
        mma_m16n8k16_bf16(s[2 * np], qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3], k0_, k1_);
        mma_m16n8k16_bf16(s[2 * np + 1], qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3], k2_, k3_);
        mma_m16n8k16_bf16(dp[2 * np], oa[kk][0], oa[kk][1], oa[kk][2], oa[kk][3], v0, v1);
        mma_m16n8k16_bf16(dp[2 * np + 1], oa[kk][0], oa[kk][1], oa[kk][2], oa[kk][3], v2, v3);
      }
    }
    // dS = c P (dP - E), rows = queries, columns = keys
    uint32_t da[2][4];
#pragma unroll
    for (int n = 0; n < 4; ++n) {
      float ds[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int hr = e >> 1;
        const int r = hr ? row_b : row_a;
        const int key = kt + 8 * n + 2 * tq + (e & 1);
        const bool vis = r < p.S && key < p.S && (!p.causal || key <= r);
        const float pr = vis ? fast_exp2(s[n][e] * p.scale_log2 - lse[hr]) : 0.f;
        ds[e] = c[hr] * pr * (dp[n][e] - E[hr]);
      }
      const int ks = n >> 1, hi = n & 1;
      da[ks][2 * hi + 0] = pack_bf16x2(ds[0], ds[1]);
      da[ks][2 * hi + 1] = pack_bf16x2(ds[2], ds[3]);
    }
    // dQ += dS K: 16 rows x 128 d, K = 32 keys (K tile transposed)
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
#pragma unroll
      for (int np = 0; np < 8; ++np) {
        const int brow = 16 * ks + ((lane >> 3) & 1) * 8 + (lane & 7);
        const int bc = 2 * np + ((lane >> 4) & 1);
        uint32_t k0_, k1_, k2_, k3_;
        ldmatrix_x4_trans(sK + sw(brow, bc), k0_, k1_, k2_, k3_);
        mma_m16n8k16_bf16(dq[2 * np], da[ks][0], da[ks][1], da[ks][2], da[ks][3], k0_, k1_);
        mma_m16n8k16_bf16(dq[2 * np + 1], da[ks][0], da[ks][1], da[ks][2], da[ks][3], k2_, k3_);
      }
    }
  }
#pragma unroll
  for (int n = 0; n < 16; ++n) {
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      const int r = hr ? row_b : row_a;
      if (r >= p.S) continue;
      const size_t off = ((static_cast<size_t>(b) * p.S + r) * p.Hq + hq) * HD + 8 * n + 2 * tq;
      *reinterpret_cast<uint32_t*>(p.dq + off) = pack_bf16x2(dq[n][2 * hr] * p.scale, dq[n][2 * hr + 1] * p.scale);
    }
  }
}

}  // namespace bwd

cudaError_t launch_backward(const __nv_bfloat16* q, const __nv_bfloat16* k, const __nv_bfloat16* v,
                            const float* lambda, const __nv_bfloat16* o_branch, const float* lse,
                            const __nv_bfloat16* dout, __nv_bfloat16* dq, __nv_bfloat16* dk, __nv_bfloat16* dv,
                            float* dlambda, float* E, int B, int S, int Hq, int Hkv, int causal,
                            cudaStream_t stream) {
  using namespace bwd;
  const long long rows = static_cast<long long>(B) * S;
  const int n_pairs = Hq / 2;
  const long long warps = rows * n_pairs;
  preprocess_kernel<<<static_cast<unsigned>((warps + 3) / 4), 128, 0, stream>>>(dout, o_branch, E, dlambda, rows,
                                                                                  n_pairs);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  Params p;
  p.q = q;
  p.k = k;
  p.v = v;
  p.dout = dout;
  p.lambda = lambda;
  p.lse = lse;
  p.E = E;
  p.dq = dq;
  p.dk = dk;
  p.dv = dv;
  p.B = B;
  p.S = S;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.causal = causal;
  p.scale = 1.f / sqrtf(static_cast<float>(HD));
  p.scale_log2 = 1.4426950408889634f * p.scale;
  e = cudaFuncSetAttribute(dkdv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kDkdvSmem);
  if (e != cudaSuccess) return e;
  dkdv_kernel<<<dim3((S + kKvRows - 1) / kKvRows, Hkv, B), 128, kDkdvSmem, stream>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  dq_kernel<<<dim3((S + kQTile - 1) / kQTile, Hq, B), 128, kDqSmem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace da2
