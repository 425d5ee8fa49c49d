// decode_sm100.cu -- bf16 DiffAttn V2 decode step: split-KV streaming kernel with a fused combine.
//
// Operator ("Differential Attention (V2)" lesson, "The differential concept" and "V1 vs V2";
// pairing per "Differential Transformer V2 soll KI-Training stabiler machen", shared-KV
// section): for the new token of sequence b and pair p (heads 2p, 2p+1, KV head g)
//   out[b,p] = softmax(q1 K^T/sqrt(D)) V - lambda[b,p] softmax(q2 K^T/sqrt(D)) V
// over the cached keys [0, seqlens[b]), or for a sliding-window layer over the last `window`
// of them (the window of the "Attention variants" lesson's sliding-window step).
//
// Decode is bound by HBM bandwidth: every visible K/V row must be read once, and V2 reads
// it once for BOTH branches and for every query head of the GQA group (the group's query
// heads are all pairs that share KV head g). Design:
//
//  * Grid (split, g, b). A CTA streams keys [base + split*L, min(base + (split+1)*L, seqlen))
//    of KV head g (base = 0, or with a window the 64-token stage boundary at or below its
//    first key, so keys before the window are not read) through a 3-stage shared-memory
//    ring filled by TMA (64 tokens x 128 d of K and of V
//    per stage, 128-byte swizzled so ldmatrix reads are bank-conflict free). Two CTAs fit
//    on an SM, so up to 6 stages (192 KB) per SM are in flight.
//  * Four consumer warps each take 16 tokens of every stage and compute, on the legacy
//    warp-level tensor-core path (mma.sync m16n8k16, bf16 in, fp32 accumulate),
//      S^T[16 tok x 8 heads] = K[16 x 128] . Q^T[128 x 8]         (N = 8 = the group's heads)
//      O^T[128 x 8 heads]   += V^T[128 x 16] . P^T[16 x 8]
//    P^T is the S^T accumulator fragment transposed in registers with movmatrix, so the
//    probabilities never touch shared memory. Each thread holds both heads of one pair.
//  * Online softmax per head in the log2 domain. Each warp keeps its own (m, l, O^T); at
//    the end of the CTA the four warps merge through shared memory and write one partial
//    (m, l, O unnormalised) per head and split to the workspace.
//  * Combine, fused: each working split of (b, g) counts itself on a per-(b, g) counter
//    once its partials are visible device-wide; the split that completes the count merges
//    all splits of the group's pairs with the log-sum-exp rule (one warp per pair) and
//    writes O1/L1 - lambda O2/L2, rounded once to bf16. No second kernel, no launch gap.
//
// The grid is sized from Smax on the host; CTAs whose split starts past seqlens[b] return
// at once (split 0 of an empty sequence writes its zero output) and the merge reads only the
// splits that exist, so no host sync is needed. The counters are zeroed on the stream
// before each launch.

#include "bounds.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace da2 {
namespace decode {

#ifdef DA2_DEBUG_BOUNDS
// Test hook of the debug build: when nonzero, CTA (0, 0, 0) announces but never issues the
// copies of its ring stage number g_withhold_stage - 1, so that its consumers' bounded waits
// expire and the kernel leaves through its abort path (set by diffattn_v2_test_withhold_decode_stage).
__device__ int g_withhold_stage = 0;
#endif

constexpr int HD = 128;
constexpr int kTok = 64;                              // tokens per stage
constexpr int kStages = 3;
constexpr int kConsumerWarps = 4;
constexpr int kThreads = 32 * (kConsumerWarps + 1);   // + 1 TMA producer warp
constexpr uint32_t kHalfBytes = kTok * 64 * 2;        // 64 tokens x 64 d bf16 = 8 KB
constexpr uint32_t kStageBytes = 4 * kHalfBytes;      // K lo/hi + V lo/hi = 32 KB
constexpr uint32_t kOffBar = kStages * kStageBytes;
constexpr uint32_t kOffMisc = kOffBar + 8 * 2 * kStages;
constexpr uint32_t kOffPages = kOffMisc + 16;                // page indices of a paged split
constexpr int kMaxSplitPages = 512;                           // split_len (<= 4096) / page_size (>= 8)
constexpr uint32_t kSmemUsed = kOffPages + 4 * kMaxSplitPages;
constexpr uint32_t kSmemBytes = kSmemUsed + 1024;

struct Params {
  const __nv_bfloat16* q;   // [B,Hq,D]
  const int32_t* seqlens;   // [B]
  float* ws_o;              // [B,T,Hq,nsplit,D]
  float* ws_ml;             // [B,T,Hq,nsplit,2]
  int* counters;            // [B,Hkv] working splits done, zero at launch
  const float* lambda;      // [B,T,Hq/2]
  __nv_bfloat16* out;       // [B,T,Hq/2,D]
  int* err;
  int B, Smax, Hq, Hkv, nsplit, split_len;
  int T;                    // new tokens per sequence (1: plain decode); T * group <= 16
  int window;               // T == 1: the token sees only keys seqlen-window .. seqlen-1 (0: all)
  float scale_log2;
  // paged caches [num_pages, page_size, Hkv, D]: logical token t of sequence b is row
  // t % page_size of page block_table[b * max_pages + t / page_size]; null = [B, Smax] caches
  const int32_t* block_table;
  int max_pages, page_shift, box_tok;  // page_size = 1 << page_shift; tokens per TMA box
};

// One warp merges the splits of both heads of `pair` for row bt = b * T + token and writes
// O1/L1 - lambda O2/L2. Splits past the token's visible keys hold (m = -inf, l = 0, O = 0) and
// weigh 0. The partials were written by other CTAs of this grid: they are read through L2.
__device__ __forceinline__ void combine_pair(const Params& p, int bt, int pair, int ns, int lane) {
  const int n_pairs = p.Hq >> 1;
  const size_t n_rows = static_cast<size_t>(p.B) * p.T * p.Hq * p.nsplit;  // partial rows of the workspace
  if (!checked(bt < p.B * p.T && pair < n_pairs && ns <= p.nsplit &&
                   (static_cast<size_t>(bt) * p.Hq + 2 * pair + 1) * p.nsplit + ns <= n_rows, p.err))
    return;
  float res[2][4];
#pragma unroll
  for (int br = 0; br < 2; ++br) {
    const size_t row0 = (static_cast<size_t>(bt) * p.Hq + 2 * pair + br) * p.nsplit;
    float M = -INFINITY;
    for (int s = lane; s < ns; s += 32) M = fmaxf(M, __ldcg(p.ws_ml + (row0 + s) * 2));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    const float Mu = (M == -INFINITY) ? 0.f : M;
    float L = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s = 0; s < ns; ++s) {
      const float2 ml = __ldcg(reinterpret_cast<const float2*>(p.ws_ml) + row0 + s);
      const float sc = fast_exp2(ml.x - Mu);
      L += ml.y * sc;
      const float4 v = __ldcg(reinterpret_cast<const float4*>(p.ws_o + (row0 + s) * HD) + lane);
      acc.x += v.x * sc;
      acc.y += v.y * sc;
      acc.z += v.z * sc;
      acc.w += v.w * sc;
    }
    const float inv = (L > 0.f) ? 1.f / L : 0.f;
    res[br][0] = __fmul_rn(acc.x, inv);
    res[br][1] = __fmul_rn(acc.y, inv);
    res[br][2] = __fmul_rn(acc.z, inv);
    res[br][3] = __fmul_rn(acc.w, inv);
  }
  const float lam = __ldg(p.lambda + static_cast<size_t>(bt) * n_pairs + pair);
  uint2 packed;
  packed.x = pack_bf16x2(__fmaf_rn(-lam, res[1][0], res[0][0]), __fmaf_rn(-lam, res[1][1], res[0][1]));
  packed.y = pack_bf16x2(__fmaf_rn(-lam, res[1][2], res[0][2]), __fmaf_rn(-lam, res[1][3], res[0][3]));
  reinterpret_cast<uint2*>(p.out + (static_cast<size_t>(bt) * n_pairs + pair) * HD)[lane] = packed;
}

// NT = number of 8-head column tiles per group (1 for group size <= 8, 2 for 16).
template <int NT>
__global__ void __launch_bounds__(kThreads, 2)
diffattn_decode_split(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                      const Params p) {
  // The MMA's N dimension holds the (new token, query head) columns of the group: column
  // n is token n / group, head n % group; q is [B,T,Hq,D] and the partials are per column.
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  auto full = [&](int s) -> uint32_t { return sbase + kOffBar + 8u * s; };
  auto empty = [&](int s) -> uint32_t { return sbase + kOffBar + 8u * (kStages + s); };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc);

  const int split = blockIdx.x;
  const int g = blockIdx.y;
  const int b = blockIdx.z;
  const int group = p.Hq / p.Hkv;
  const int seqlen = min(max(__ldg(p.seqlens + b), 0), p.Smax);
  // with a sliding window the visible keys start at lo; the splits then start at the stage
  // boundary below it, so the keys before the window are never read
  const int lo = p.window > 0 ? max(0, seqlen - p.window) : 0;
  const int base = lo / kTok * kTok;
  const int t0 = base + split * p.split_len;
  if (t0 >= seqlen) {  // uniform for the CTA: nothing to read
    if (split == 0) {
      // an empty sequence has no working split to merge it: its outputs are zero
      const int pairs_g = group >> 1, n_pairs = p.Hq >> 1;
      for (int i = threadIdx.x; i < p.T * pairs_g * (HD / 8); i += blockDim.x) {
        const int c = i % (HD / 8), r = i / (HD / 8);
        const int pair = g * pairs_g + r % pairs_g;
        if (checked(pair < n_pairs && r / pairs_g < p.T, p.err))
          reinterpret_cast<uint4*>(p.out + (static_cast<size_t>(b) * p.T + r / pairs_g) * n_pairs * HD +
                                   static_cast<size_t>(pair) * HD)[c] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
    return;
  }
  const int t1 = min(t0 + p.split_len, seqlen);
  const int n_stages = (t1 - t0 + kTok - 1) / kTok;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), kConsumerWarps);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kConsumerWarps) {
    // --------------------------------------------------------------------- producer
    int* pages = reinterpret_cast<int*>(smem + kOffPages);
    const int page_size = 1 << p.page_shift;
    const int first_page = t0 >> p.page_shift;
    if (p.block_table) {
      // the split's page indices, read once: logical pages first_page .. (t1-1) / page_size
      const int n_pages = ((t1 - 1) >> p.page_shift) - first_page + 1;
      for (int i = lane; i < n_pages; i += 32)
        if (checked(i < kMaxSplitPages && first_page + i < p.max_pages, p.err))
          pages[i] = __ldg(p.block_table + static_cast<size_t>(b) * p.max_pages + first_page + i);
      __syncwarp();
    }
    if (lane == 0) {
      int issued = 0;
      for (int i = 0; i < n_stages; ++i) {
        const int s = i % kStages;
        const uint32_t ph = (i / kStages) & 1;
        if (!mbar_wait(empty(s), ph ^ 1, abort_flag)) break;
        const uint32_t dst = sbase + s * kStageBytes;
        const int tok = t0 + i * kTok;
        mbar_arrive_expect_tx(full(s), kStageBytes);
        // skipped on a violation: the stage's barrier stays short and the consumers give up
        if (!checked(within(dst, kStageBytes, sbase, kOffBar) && g < p.Hkv, p.err)) continue;
#ifdef DA2_DEBUG_BOUNDS
        if (g_withhold_stage == i + 1 && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0) continue;
#endif
        if (!p.block_table) {
          tma_load_4d(dst + 0 * kHalfBytes, &tmK, full(s), 0, g, tok, b);
          tma_load_4d(dst + 1 * kHalfBytes, &tmK, full(s), 64, g, tok, b);
          tma_load_4d(dst + 2 * kHalfBytes, &tmV, full(s), 0, g, tok, b);
          tma_load_4d(dst + 3 * kHalfBytes, &tmV, full(s), 64, g, tok, b);
        } else {
          // one box per page (or per 64 tokens of a larger page); a box's rows land at the
          // same smem rows a single 64-token box would fill, so the swizzle is unchanged.
          // Tokens past the sequence read page -1: out of range, filled with zeros.
          for (int sb = 0; sb < kTok; sb += p.box_tok) {
            const int tk = tok + sb;
            const int pi = (tk >> p.page_shift) - first_page;
            const int page = (tk < t1 && checked(pi >= 0 && pi < kMaxSplitPages, p.err)) ? pages[pi] : -1;
            const int row = tk & (page_size - 1);
            const uint32_t o = static_cast<uint32_t>(sb) * 128u;
            tma_load_4d(dst + 0 * kHalfBytes + o, &tmK, full(s), 0, g, row, page);
            tma_load_4d(dst + 1 * kHalfBytes + o, &tmK, full(s), 64, g, row, page);
            tma_load_4d(dst + 2 * kHalfBytes + o, &tmV, full(s), 0, g, row, page);
            tma_load_4d(dst + 3 * kHalfBytes + o, &tmV, full(s), 64, g, row, page);
          }
        }
        issued = i + 1;
      }
      if (*abort_flag) {
        // let every issued copy land before the CTA's shared memory is released; each wait has
        // its own time limit (a wait that gives up must not end the ones after it)
        for (int i = max(0, issued - kStages); i < issued; ++i) {
          volatile int no_abort = 0;
          mbar_wait(full(i % kStages), (i / kStages) & 1, &no_abort);
        }
      }
    }
    // the producer warp takes part in the final merge barrier only through __syncthreads
  }

  // ------------------------------------------------------------------------ consumers
  const int gl = lane >> 2;  // fragment row group
  const int tq = lane & 3;   // fragment column pair
  float o[NT][8][4];
  float m_run[NT][2], l_part[NT][2];
  if (warp < kConsumerWarps) {
    // Q^T as B fragments: column n = 8 nt + gl (token n / group, head n % group), k = d
    uint32_t qf[NT][8][2];
    const int hq0 = g * group;  // first query head of the group
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int n = nt * 8 + gl;
      const bool hv = n < p.T * group;
      const int tok = hv ? n / group : 0, h = hv ? n % group : 0;
      checked(hq0 + h < p.Hq && tok < p.T, p.err);  // q row inside [B, T, Hq]
      const uint32_t* qrow =
          reinterpret_cast<const uint32_t*>(p.q + ((static_cast<size_t>(b) * p.T + tok) * p.Hq + hq0 + h) * HD);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        qf[nt][kk][0] = hv ? __ldg(qrow + (16 * kk + 2 * tq) / 2) : 0u;
        qf[nt][kk][1] = hv ? __ldg(qrow + (16 * kk + 2 * tq + 8) / 2) : 0u;
      }
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      m_run[nt][0] = m_run[nt][1] = -INFINITY;
      l_part[nt][0] = l_part[nt][1] = 0.f;
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) o[nt][mt][0] = o[nt][mt][1] = o[nt][mt][2] = o[nt][mt][3] = 0.f;
    }

    // per-lane ldmatrix row/chunk selectors
    const int k_row = 16 * warp + (lane & 7) + ((lane >> 3) & 1) * 8;    // K: matrices (r0,k0)(r8,k0)(r0,k8)(r8,k8)
    const int k_csel = (lane >> 4) & 1;
    const int v_row = 16 * warp + (lane & 7) + ((lane >> 4) & 1) * 8;    // V: matrices (t0,d0)(t0,d8)(t8,d0)(t8,d8)
    const int v_csel = (lane >> 3) & 1;

    for (int i = 0; i < n_stages; ++i) {
      const int s = i % kStages;
      const uint32_t ph = (i / kStages) & 1;
      // the warp leaves together: the loop body is made of warp-collective instructions
      if (!__all_sync(0xffffffffu, mbar_wait(full(s), ph, abort_flag))) break;
      const uint32_t kb = sbase + s * kStageBytes;
      const uint32_t vb = kb + 2 * kHalfBytes;

      float sacc[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) sacc[nt][0] = sacc[nt][1] = sacc[nt][2] = sacc[nt][3] = 0.f;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const int chunk = 2 * kk + k_csel;  // 16-byte chunk of d
        const uint32_t addr = kb + (chunk >> 3) * kHalfBytes + k_row * 128 + (((chunk & 7) ^ (k_row & 7)) << 4);
        uint32_t a0, a1, a2, a3;
        ldmatrix_x4(addr, a0, a1, a2, a3);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) mma_m16n8k16_bf16(sacc[nt], a0, a1, a2, a3, qf[nt][kk][0], qf[nt][kk][1]);
      }

      // scale, mask tokens outside [t0, t1), online softmax per head column
      const int tok_a = t0 + i * kTok + 16 * warp + gl;
      const int tok_b = tok_a + 8;
      uint32_t pb[NT][2];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        // this thread's two columns belong to one new token, which sees keys below
        // seqlen - T + token + 1 (causal among the new tokens)
        const int col_tok = (8 * nt + 2 * tq) / group;
        const int lim = col_tok < p.T ? min(t1, seqlen - p.T + col_tok + 1) : t1;
        const bool va = tok_a < lim && tok_a >= lo, vb_ = tok_b < lim && tok_b >= lo;
        float x[4];
        x[0] = va ? sacc[nt][0] * p.scale_log2 : -INFINITY;
        x[1] = va ? sacc[nt][1] * p.scale_log2 : -INFINITY;
        x[2] = vb_ ? sacc[nt][2] * p.scale_log2 : -INFINITY;
        x[3] = vb_ ? sacc[nt][3] * p.scale_log2 : -INFINITY;
        float pr[4];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          float mx = fmaxf(x[c], x[c + 2]);
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
          const float m_new = fmaxf(m_run[nt][c], mx);
          const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
          const float alpha = fast_exp2(m_run[nt][c] - m_use);
          m_run[nt][c] = m_new;
          pr[c] = fast_exp2(x[c] - m_use);
          pr[c + 2] = fast_exp2(x[c + 2] - m_use);
          l_part[nt][c] = l_part[nt][c] * alpha + pr[c] + pr[c + 2];
#pragma unroll
          for (int mt = 0; mt < 8; ++mt) {
            o[nt][mt][c] *= alpha;
            o[nt][mt][c + 2] *= alpha;
          }
        }
        // P^T fragments: transpose the two 8x8 (token x head) blocks
        pb[nt][0] = movmatrix_trans(pack_bf16x2(pr[0], pr[1]));
        pb[nt][1] = movmatrix_trans(pack_bf16x2(pr[2], pr[3]));
      }

#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        const int chunk = 2 * mt + v_csel;
        const uint32_t addr = vb + (chunk >> 3) * kHalfBytes + v_row * 128 + (((chunk & 7) ^ (v_row & 7)) << 4);
        uint32_t a0, a1, a2, a3;
        ldmatrix_x4_trans(addr, a0, a1, a2, a3);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) mma_m16n8k16_bf16(o[nt][mt], a0, a1, a2, a3, pb[nt][0], pb[nt][1]);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty(s));
    }
    // full row sums of this warp: reduce the per-thread partials over the 8 token rows
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        float v = l_part[nt][c];
        v += __shfl_xor_sync(0xffffffffu, v, 4);
        v += __shfl_xor_sync(0xffffffffu, v, 8);
        v += __shfl_xor_sync(0xffffffffu, v, 16);
        l_part[nt][c] = v;
      }
  }

  // every TMA write has landed (consumers waited on every full barrier) -> reuse the ring
  __syncthreads();
  const bool aborted = *abort_flag != 0;
  float* w_o = reinterpret_cast<float*>(smem);                        // [warp][8*NT heads][D]
  float* w_ml = w_o + kConsumerWarps * 8 * NT * HD;                    // [warp][8*NT][2]
  if (warp < kConsumerWarps && !aborted) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int h = nt * 8 + 2 * tq + (c & 1);
          const int d = 16 * mt + gl + (c >> 1) * 8;
          w_o[(warp * 8 * NT + h) * HD + d] = o[nt][mt][c];
        }
      }
      if (gl == 0) {
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int h = nt * 8 + 2 * tq + c;
          w_ml[(warp * 8 * NT + h) * 2 + 0] = m_run[nt][c];
          w_ml[(warp * 8 * NT + h) * 2 + 1] = l_part[nt][c];
        }
      }
    }
  }
  __syncthreads();
  if (aborted) {
    if (threadIdx.x == 0) atomicCAS(p.err, 0, kErrDecodeWait);
    return;
  }
  if (warp < kConsumerWarps) {
    const int d = threadIdx.x;  // 0..127
    const int nh = min(p.T * group, 8 * NT);
    for (int h = 0; h < nh; ++h) {  // h: column (token h / group, head h % group)
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, w_ml[(w * 8 * NT + h) * 2]);
      const float Mu = (M == -INFINITY) ? 0.f : M;
      float O = 0.f, L = 0.f;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) {
        const float sc = fast_exp2(w_ml[(w * 8 * NT + h) * 2] - Mu);
        O += w_o[(w * 8 * NT + h) * HD + d] * sc;
        L += w_ml[(w * 8 * NT + h) * 2 + 1] * sc;
      }
      const size_t row =
          ((static_cast<size_t>(b) * p.T + h / group) * p.Hq + g * group + h % group) * p.nsplit + split;
      if (!checked(row < static_cast<size_t>(p.B) * p.T * p.Hq * p.nsplit, p.err)) continue;
      p.ws_o[row * HD + d] = O;
      if (d == 0) {
        p.ws_ml[row * 2 + 0] = M;
        p.ws_ml[row * 2 + 1] = L;
      }
    }
  }

  // ---- fused combine: count this split once its partials are visible device-wide; the
  // split that completes the count for (b, g) merges the group's pairs
  __threadfence();
  __syncthreads();
  volatile int* last_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);
  const int ns = (seqlen - base + p.split_len - 1) / p.split_len;  // working splits of sequence b
  if (threadIdx.x == 0)
    *last_flag = (checked(b < p.B && g < p.Hkv && ns <= p.nsplit, p.err) &&
                  atomicAdd(p.counters + static_cast<size_t>(b) * p.Hkv + g, 1) == ns - 1) ? 1 : 0;
  __syncthreads();
  if (!*last_flag) return;
  __threadfence();  // the other splits' partials, counted before ours, are visible
  const int pairs_g = group >> 1;
  for (int item = warp; item < p.T * pairs_g; item += kConsumerWarps + 1)
    combine_pair(p, b * p.T + item / pairs_g, g * pairs_g + item % pairs_g, ns, lane);
}

}  // namespace decode

#ifdef DA2_DEBUG_BOUNDS
extern "C" __attribute__((visibility("default"))) int diffattn_v2_test_withhold_decode_stage(int stage_plus_one) {
  return cudaMemcpyToSymbol(decode::g_withhold_stage, &stage_plus_one, sizeof(int)) == cudaSuccess ? 0 : -3;
}
#endif

cudaError_t launch_decode(const CUtensorMap& tmK, const CUtensorMap& tmV, const __nv_bfloat16* q,
                          const int32_t* seqlens, const float* lambda, __nv_bfloat16* out, float* ws_o,
                          float* ws_ml, int* counters, int* err, int B, int Smax, int Hq, int Hkv, int nsplit,
                          int split_len, const int32_t* block_table, int max_pages, int page_shift, int T,
                          cudaStream_t stream, int window) {
  using namespace decode;
  Params p;
  p.q = q;
  p.seqlens = seqlens;
  p.ws_o = ws_o;
  p.ws_ml = ws_ml;
  p.counters = counters;
  p.lambda = lambda;
  p.out = out;
  p.err = err;
  p.B = B;
  p.Smax = Smax;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.nsplit = nsplit;
  p.split_len = split_len;
  p.scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(HD));
  p.T = T;
  p.window = window;
  p.block_table = block_table;
  p.max_pages = max_pages;
  p.page_shift = page_shift;
  p.box_tok = block_table ? min(1 << page_shift, kTok) : kTok;
  const int group = Hq / Hkv;
  dim3 grid(nsplit, Hkv, B);
  cudaError_t e = cudaMemsetAsync(counters, 0, static_cast<size_t>(B) * Hkv * sizeof(int), stream);
  if (e != cudaSuccess) return e;
  if (T * group > 8) {
    e = cudaFuncSetAttribute(diffattn_decode_split<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    diffattn_decode_split<2><<<grid, kThreads, kSmemBytes, stream>>>(tmK, tmV, p);
  } else {
    e = cudaFuncSetAttribute(diffattn_decode_split<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    diffattn_decode_split<1><<<grid, kThreads, kSmemBytes, stream>>>(tmK, tmV, p);
  }
  return cudaGetLastError();
}

}  // namespace da2
