// backward_sm100.cu -- gradients of the bf16 DiffAttn V2 prefill on the 5th-generation tensor
// cores (sm_100a).
//
// Chain rule of out = A_1 V - lambda A_2 V, A_b = softmax(Q_b K^T / sqrt(D)) ("Differential
// Attention (V2)" lesson, "The differential concept"; causal mask of the "Attention variants"
// lesson), per pair of heads (2p, 2p+1) over KV head g, with dO the upstream gradient:
//   dP   = dO V^T                       (one product per pair: both branches read dO and V)
//   W    = A_1 - lambda A_2             (the combined weights, rounded to bf16 once)
//   dS_1 = A_1 (dP - E_1),  dS_2 = -lambda A_2 (dP - E_2),   E_b = dO . O_b per row
//   dV  += W^T dO,   dK += (dS_1^T Q_1 + dS_2^T Q_2) / sqrt(D),   dQ_b = dS_b K / sqrt(D)
//   dlambda = -dO . O_2
// A_b is recomputed from the forward's base-2 row log-sum-exp: A_b = 2^(s log2(e)/sqrt(D) - lse_b).
//
// Three launches, no atomics (the result is deterministic):
//   preprocess   one warp per (token, pair): E_1, E_2, dlambda, and the row terms the other
//                kernels stream, negated and stored per 64-row block as five arrays of 64
//                fp32 (-lse_1, -lse_2, -E_1, -E_2, -lambda); rows past S (to a multiple of
//                128) get -lse = -inf so their probabilities are exactly 0 without
//                per-element row checks
//   dkdv_sm100   a CTA owns 128 keys of one KV head (the TMEM lanes) and walks every pair of
//                the group and every 64-row query block that sees the keys
//   dq_sm100     a CTA owns 128 query rows of one pair (the TMEM lanes) and walks the 64-key
//                blocks they see
// Both tile kernels have the forward prefill's shape: a TMA producer warp, an MMA warp (one
// thread issues tcgen05.mma), 8 elementwise warps that read fp32 scores from TMEM and write
// bf16 operands back over them. A step's scores are produced in two 32-column halves so that
// the elementwise work on one half overlaps the MMAs of the other.

#include "bounds.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace da2 {
namespace bwd_tc {

constexpr int HD = 128;
constexpr int kStages = 2;

// Elementwise warps: 8 (each thread takes 32 columns of a step) or 16 (16 columns). Warps
// w and w+4k read the same TMEM lanes (w % 4 picks the lane quarter) and split the columns.
#ifndef DA2_BWD_EW_WARPS
#define DA2_BWD_EW_WARPS 8
#endif
constexpr int kEwWarps = DA2_BWD_EW_WARPS;
static_assert(kEwWarps == 8 || kEwWarps == 16, "elementwise warps");
constexpr int kGroups = kEwWarps / 4;      // column groups of a 64-column step
constexpr int kCols = 64 / kGroups;        // columns per elementwise thread
// Pipeline chains per step: the score MMAs of a chain cover 64 / kChains columns (their N)
// and are committed together; the groups of a chain turn them into operands together.
#ifndef DA2_BWD_CHAINS
#define DA2_BWD_CHAINS 1
#endif
constexpr int kChains = DA2_BWD_CHAINS;
static_assert(kChains >= 1 && kGroups % kChains == 0, "chains");
constexpr int kChainCols = 64 / kChains;
constexpr int kGroupsPerChain = kGroups / kChains;
constexpr int kProducerWarp = kEwWarps;
constexpr int kMmaWarp = kEwWarps + 1;
constexpr int kThreads = 32 * (kEwWarps + 2);

// Per chain: the MMA warp issues the chain's scores, the four warps of each of its column
// groups turn them into bf16 operands written (two per 32-bit column) over the first half of
// the group's own fp32 columns, and the MMA warp accumulates from them. TMEM column of the
// bf16 operands of the 16 columns from column q (a K-step of an accumulation MMA):
__host__ __device__ constexpr uint32_t operand_col(int q) {
  return static_cast<uint32_t>((q / kCols) * kCols + (q % kCols) / 2);
}
constexpr int kStatArrays = 5;                 // -lse1, -lse2, -E1, -E2, -lambda
constexpr int kStatBlock = 64;                 // rows per block of the five arrays
constexpr int kRowPad = 128;                   // stats rows padded to a multiple of this

constexpr uint32_t kIdescS = idesc_bf16_f32(128, kChainCols, false);  // scores: N = one chain's columns
constexpr uint32_t kIdescAcc = idesc_bf16_f32(128, 128, true);  // accumulators: B MN-major, N = d

// TMEM columns. kTmA holds one resident 128 x 128 operand (bf16 pairs) read as the A
// operand of a score MMA: K in the dK/dV kernel, Q_1 in the dQ kernel.
constexpr uint32_t kTmS1 = 0, kTmS2 = 64, kTmDP = 128, kTmA = 192, kTmAcc0 = 256, kTmAcc1 = 384;

// K-major SW128 operand of R rows: K-step kk (16 of d) -> chunk kk/4, +32 bytes per 16 elements
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t base, uint32_t chunk_bytes, int kk) {
  return sdesc_sw128(base + (kk >> 2) * chunk_bytes + (kk & 3) * 32, 16, 1024);
}
// MN-major SW128 B operand (rows = reduction dim, d = N): K-step of 16 rows from `row`
__device__ __forceinline__ uint64_t desc_mnmajor(uint32_t base, uint32_t chunk_bytes, int row) {
  return sdesc_sw128(base + row * 128, chunk_bytes, 1024);
}

struct Params {
  const float* stats;        // [B, Hq/2, S_pad/64, 5, 64]
  __nv_bfloat16* dq;         // [B,S,Hq,D]
  __nv_bfloat16* dk;         // [B,S,Hkv,D]
  __nv_bfloat16* dv;
  int* err;
  int B, S, S_pad, Hq, Hkv, causal;
  int window;                // causal sliding window: query i sees keys i-window+1 .. i (0: none)
  int n_tiles;               // 128-row tiles
  const int* cu_seqlens;     // packed sequences: sequence b is rows cu[b] .. cu[b+1]-1 (null: [B,S])
  const int* pad_off;        // packed sequences: first row of sequence b in the row terms (128-aligned)
  float scale, scale_log2;
};

// ------------------------------------------------------------------------ preprocess
// Offset of row i's term k in the stats of (b, pair).
__host__ __device__ __forceinline__ size_t stat_index(size_t bp, int S_pad, int i, int k) {
  return (bp * (S_pad / kStatBlock) + i / kStatBlock) * (kStatArrays * kStatBlock) + k * kStatBlock + i % kStatBlock;
}

__global__ void __launch_bounds__(128)
preprocess_kernel(const __nv_bfloat16* __restrict__ dout, const __nv_bfloat16* __restrict__ o_branch,
                  const float* __restrict__ lse, const float* __restrict__ lambda, float* __restrict__ stats,
                  float* __restrict__ dlam, int B, int S, int S_pad, int n_pairs) {
  const long long w = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (w >= static_cast<long long>(B) * S_pad * n_pairs) return;
  // warp w: row i of pair p of batch b, rows fastest
  const int i = static_cast<int>(w % S_pad);
  const long long bp = w / S_pad;
  const int p = static_cast<int>(bp % n_pairs);
  const int b = static_cast<int>(bp / n_pairs);
  if (i >= S) {
    if (lane < kStatArrays) stats[stat_index(bp, S_pad, i, lane)] = lane < 2 ? -INFINITY : 0.f;
    return;
  }
  const long long row = static_cast<long long>(b) * S + i;
  const uint2 g = __ldg(reinterpret_cast<const uint2*>(dout + (row * n_pairs + p) * HD) + lane);
  const float2 g0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&g.x));
  const float2 g1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&g.y));
  float e[2];
#pragma unroll
  for (int br = 0; br < 2; ++br) {
    const uint2 o = __ldg(reinterpret_cast<const uint2*>(o_branch + (row * (2 * n_pairs) + 2 * p + br) * HD) + lane);
    const float2 o0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&o.x));
    const float2 o1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&o.y));
    float v = g0.x * o0.x + g0.y * o0.y + g1.x * o1.x + g1.y * o1.y;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    e[br] = v;
  }
  if (lane < kStatArrays) {
    float t;
    if (lane < 2) t = -__ldg(lse + row * (2 * n_pairs) + 2 * p + lane);
    else if (lane < 4) t = -e[lane - 2];
    else t = -__ldg(lambda + row * n_pairs + p);
    stats[stat_index(bp, S_pad, i, lane)] = t;
  }
  if (lane == 0) dlam[row * n_pairs + p] = -e[1];
}

// Packed sequences: sequence b's row terms start at pad_off[b], each sequence padded to a
// multiple of 128 rows (pad_off[B] = the padded total). One thread: the scan is over B.
__global__ void pad_offsets_kernel(const int* __restrict__ cu, int* __restrict__ pad_off, int B) {
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    int acc = 0;
    for (int b = 0; b < B; ++b) {
      pad_off[b] = acc;
      acc += (cu[b + 1] - cu[b] + kRowPad - 1) / kRowPad * kRowPad;
    }
    pad_off[B] = acc;
  }
}

// The preprocess for packed sequences: warp w is padded row pr of pair p (rows of all pairs
// laid out as one batch of S_pad rows). Rows past a sequence's end, and past the padded
// total, get -lse = -inf.
__global__ void __launch_bounds__(128)
preprocess_varlen_kernel(const __nv_bfloat16* __restrict__ dout, const __nv_bfloat16* __restrict__ o_branch,
                         const float* __restrict__ lse, const float* __restrict__ lambda, float* __restrict__ stats,
                         float* __restrict__ dlam, const int* __restrict__ cu, const int* __restrict__ pad_off, int B,
                         int S_pad, int n_pairs) {
  const long long w = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (w >= static_cast<long long>(S_pad) * n_pairs) return;
  const int pr = static_cast<int>(w % S_pad);
  const int p = static_cast<int>(w / S_pad);
  // the sequence whose padded rows hold pr: last b with pad_off[b] <= pr (b = B: past the end)
  int lo = 0, hi = B;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(pad_off + mid) <= pr) lo = mid; else hi = mid - 1;
  }
  const int b = lo;
  const int i = pr - (b < B ? __ldg(pad_off + b) : 0);
  if (b >= B || i >= __ldg(cu + b + 1) - __ldg(cu + b)) {
    if (lane < kStatArrays) stats[stat_index(p, S_pad, pr, lane)] = lane < 2 ? -INFINITY : 0.f;
    return;
  }
  const long long row = static_cast<long long>(__ldg(cu + b)) + i;
  const uint2 g = __ldg(reinterpret_cast<const uint2*>(dout + (row * n_pairs + p) * HD) + lane);
  const float2 g0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&g.x));
  const float2 g1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&g.y));
  float e[2];
#pragma unroll
  for (int br = 0; br < 2; ++br) {
    const uint2 o = __ldg(reinterpret_cast<const uint2*>(o_branch + (row * (2 * n_pairs) + 2 * p + br) * HD) + lane);
    const float2 o0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&o.x));
    const float2 o1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&o.y));
    float v = g0.x * o0.x + g0.y * o0.y + g1.x * o1.x + g1.y * o1.y;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    e[br] = v;
  }
  if (lane < kStatArrays) {
    float t;
    if (lane < 2) t = -__ldg(lse + row * (2 * n_pairs) + 2 * p + lane);
    else if (lane < 4) t = -e[lane - 2];
    else t = -__ldg(lambda + row * n_pairs + p);
    stats[stat_index(p, S_pad, pr, lane)] = t;
  }
  if (lane == 0) dlam[row * n_pairs + p] = -e[1];
}

// Shared-memory layouts (byte offsets from a 1024-aligned base). Both tile kernels hold
// three "fixed" tiles of 128 rows and stream 64-row tiles through a 2-stage ring.
constexpr uint32_t kFixedTile = 128 * 256;     // 128 rows x 128 bf16
constexpr uint32_t kFixedChunk = 128 * 128;    // one 64-wide d half of it
constexpr uint32_t kStreamTile = 64 * 256;     // 64 rows x 128 bf16
constexpr uint32_t kStreamChunk = 64 * 128;
constexpr uint32_t kStatBytes = kStatArrays * kStatBlock * 4;  // one 64-row block

// mbarriers
enum Bar : int {
  kFixedFull = 0,
  kXFull = 1,    // +stage
  kXEmpty = 3,   // +stage
  kSFull = 5,    // +column group: its scores are in TMEM
  kPReady = 9,   // +column group: its bf16 operands are in TMEM
  kDFull = 13,
  kDrain = 14,
  kAReady = 15,  // the resident A operand is in TMEM
  kNumBars = 16
};

// dK/dV: fixed K, V (128 keys); stream Q1, Q2, dO (64 query rows) + their 64 stat records
constexpr uint32_t kKvOffK = 0;
constexpr uint32_t kKvOffV = kFixedTile;
constexpr uint32_t kKvOffX = 2 * kFixedTile;
constexpr uint32_t kKvStage = (3 * kStreamTile + kStatBytes + 1023) / 1024 * 1024;  // tiles stay 1024-aligned
constexpr uint32_t kKvOffBar = kKvOffX + kStages * kKvStage;
constexpr uint32_t kKvSmem = kKvOffBar + 256 + 1024;

// dQ: fixed Q1, Q2, dO (128 query rows); stream K, V (64 keys)
constexpr uint32_t kQOffQ1 = 0;
constexpr uint32_t kQOffQ2 = kFixedTile;
constexpr uint32_t kQOffO = 2 * kFixedTile;
constexpr uint32_t kQOffX = 3 * kFixedTile;
constexpr uint32_t kQStage = 2 * kStreamTile;
constexpr uint32_t kQOffBar = kQOffX + kStages * kQStage;
constexpr uint32_t kQSmem = kQOffBar + 256 + 1024;
static_assert(kKvStage % 1024 == 0 && kQStage % 1024 == 0, "128-byte-swizzled tiles need 1024-byte alignment");
static_assert(kKvSmem <= 232448 && kQSmem <= 232448, "shared memory per CTA");

__device__ __forceinline__ void tmem_ld_x32_wait(uint32_t taddr, uint32_t (&r)[32]) {
  tmem_ld_32x32b_x32(taddr, r);
  tmem_ld_wait(r);
}

// Common set-up: barriers, TMEM (512 columns, by warp 9). Returns the TMEM base.
__device__ __forceinline__ uint32_t setup(uint32_t bar0, uint32_t* tmem_slot, volatile int* abort_flag, int warp) {
  if (threadIdx.x == 0) {
    for (int i = 0; i < kNumBars; ++i) {
      const uint32_t count =
          (i >= kPReady && i < kPReady + kChains) ? 128u * kGroupsPerChain : (i == kAReady ? 32u * kEwWarps : 1u);
      mbar_init(bar0 + 8u * i, count);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  return *tmem_slot;
}

__device__ __forceinline__ void teardown(uint32_t tmem, const volatile int* abort_flag, int* err, int warp) {
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag) atomicCAS(err, 0, kErrBackwardWait);
  if (warp == kMmaWarp) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Write this thread's 128 / kGroups accumulator columns of its row (TMEM) as bf16, times `mul`.
__device__ __forceinline__ void store_row(uint32_t taddr, __nv_bfloat16* dst, float mul, bool valid) {
#pragma unroll 1
  for (int c = 0; c < 128 / kGroups / 32; ++c) {
    uint32_t a[32];
    tmem_ld_x32_wait(taddr + 32 * c, a);
    if (valid) {
      uint4* d = reinterpret_cast<uint4*>(dst + 32 * c);
#pragma unroll
      for (int v = 0; v < 4; ++v)
        d[v] = make_uint4(pack_bf16x2(__uint_as_float(a[8 * v + 0]) * mul, __uint_as_float(a[8 * v + 1]) * mul),
                          pack_bf16x2(__uint_as_float(a[8 * v + 2]) * mul, __uint_as_float(a[8 * v + 3]) * mul),
                          pack_bf16x2(__uint_as_float(a[8 * v + 4]) * mul, __uint_as_float(a[8 * v + 5]) * mul),
                          pack_bf16x2(__uint_as_float(a[8 * v + 6]) * mul, __uint_as_float(a[8 * v + 7]) * mul));
    }
  }
}

// N (kCols) consecutive fp32 columns of this warp's 32 lanes; the wait completes them.
template <int N>
__device__ __forceinline__ void ld_cols(uint32_t taddr, uint32_t (&r)[N]) {
  if constexpr (N == 32) {
    tmem_ld_32x32b_x32(taddr, r);
  } else {
    tmem_ld_32x32b_x16(taddr, r);
  }
}
template <int N>
__device__ __forceinline__ void ld_cols_wait(uint32_t (&r)[N]) {
  if constexpr (N == 32) {
    tmem_ld_wait(r);
  } else {
    tmem_ld_wait16(r);
  }
}
// N = 16 or 32 consecutive 32-bit columns of this warp's 32 lanes
template <int N>
__device__ __forceinline__ void st_cols(uint32_t taddr, const uint32_t (&r)[N]) {
  if constexpr (N == 32) {
    tmem_st_32x32b_x32(taddr, r);
  } else {
    tmem_st_32x32b_x16(taddr, r);
  }
}
// N packed bf16x2 columns (N = kCols / 2)
template <int N>
__device__ __forceinline__ void st_packed(uint32_t taddr, const uint32_t (&r)[N]) {
  if constexpr (N == 16) {
    tmem_st_32x32b_x16(taddr, r);
  } else {
    tmem_st_32x32b_x8(taddr, r);
  }
}

// Copy this thread's share of a resident 128-row K-major SW128 tile (row r = TMEM lane)
// into TMEM from column kTmA on, as packed bf16 pairs along d (element 2j in the low half
// of column j): the A-operand layout of a TS MMA. Each column group takes 128 / kGroups d.
__device__ __forceinline__ void tile_to_tmem(uint32_t tile, uint32_t trow, int r, int cg) {
  constexpr int kD = 128 / kGroups;
  uint32_t v[kD / 2];
#pragma unroll
  for (int u = 0; u < kD / 8; ++u) {
    const int du = (kD / 8) * cg + u;  // 16-byte unit along d, 0..15
    const uint32_t addr = tile + (du >> 3) * kFixedChunk + r * 128 + (((du & 7) ^ (r & 7)) << 4);
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v[4 * u]), "=r"(v[4 * u + 1]), "=r"(v[4 * u + 2]), "=r"(v[4 * u + 3])
                 : "r"(addr));
  }
  st_cols(trow + kTmA + (kD / 2) * cg, v);
}

// --------------------------------------------------------------------------- dK / dV
// kVarlen: packed sequences (p.cu_seqlens); kWindow: causal sliding window (p.window). The
// plain [B,S] backward is the <false, false> instance and carries neither.
template <bool kVarlen, bool kWindow>
__global__ void __launch_bounds__(kThreads, 1)
dkdv_sm100(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmO,
           const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + kKvOffBar;
  auto bar = [&](int i) -> uint32_t { return bar0 + 8u * static_cast<uint32_t>(i); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kKvOffBar + 128);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kKvOffBar + 136);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_pairs = p.Hq >> 1, group = p.Hq / p.Hkv, gpairs = group >> 1;
  const int g = static_cast<int>(blockIdx.x) % p.Hkv;
  const int b = static_cast<int>(blockIdx.x) / p.Hkv;
  const int tile = static_cast<int>(blockIdx.y);  // tile 0 (most query blocks when causal) first
  const int k0 = tile * 128;
  // sequence extent: a [B,S] batch, or packed sequences whose tensors are one [1,T] batch
  // (tok0: the sequence's first row; tb: the batch coordinate of the tensor maps; sb, srow0:
  // where the sequence's row terms start)
  int S = p.S, tok0 = 0, tb = b, srow0 = 0;
  size_t sb = static_cast<size_t>(b) * n_pairs;
  if (kVarlen) {
    tok0 = __ldg(p.cu_seqlens + b);
    S = __ldg(p.cu_seqlens + b + 1) - tok0;
    tb = 0;
    sb = 0;
    srow0 = __ldg(p.pad_off + b);
  }
  if (k0 >= S) return;  // uniform over the CTA: the key tile lies past the sequence's end
  const size_t row_base = kVarlen ? static_cast<size_t>(tok0) : static_cast<size_t>(b) * p.S;
  const int nq = (S + 63) / 64;                     // 64-row query blocks
  const int q_first = p.causal ? k0 / 64 : 0;
  // with a window the tile's keys k0 .. k0+127 are seen by queries up to k0+127+window-1
  const int q_end = kWindow ? min(nq, (k0 + 126 + p.window) / 64 + 1) : nq;
  const int steps_per_pair = q_end - q_first;
  const int n_steps = gpairs * steps_per_pair;

  const uint32_t tmem = setup(bar0, tmem_slot, abort_flag, warp);

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmO);
      mbar_arrive_expect_tx(bar(kFixedFull), 2 * kFixedTile);
      for (int c = 0; c < 2; ++c) {
        tma_load_4d(sbase + kKvOffK + c * kFixedChunk, &tmK, bar(kFixedFull), c * 64, g, tok0 + k0, tb);
        tma_load_4d(sbase + kKvOffV + c * kFixedChunk, &tmV, bar(kFixedFull), c * 64, g, tok0 + k0, tb);
      }
      int issued = 0;
      for (int t = 0; t < n_steps; ++t) {
        const int s = t & 1;
        if (!mbar_wait(bar(kXEmpty + s), ((t >> 1) & 1) ^ 1, abort_flag)) break;
        const int pair = g * gpairs + t / steps_per_pair;
        const int q0 = (q_first + t % steps_per_pair) * 64;
        const uint32_t st = sbase + kKvOffX + s * kKvStage;
        mbar_arrive_expect_tx(bar(kXFull + s), 3 * kStreamTile + kStatBytes);
        for (int c = 0; c < 2; ++c) {
          tma_load_4d(st + c * kStreamChunk, &tmQ, bar(kXFull + s), c * 64, 2 * pair, tok0 + q0, tb);
          tma_load_4d(st + kStreamTile + c * kStreamChunk, &tmQ, bar(kXFull + s), c * 64, 2 * pair + 1, tok0 + q0, tb);
          tma_load_4d(st + 2 * kStreamTile + c * kStreamChunk, &tmO, bar(kXFull + s), c * 64, pair, tok0 + q0, tb);
        }
        bulk_load(st + 3 * kStreamTile, p.stats + stat_index(sb + pair, p.S_pad, srow0 + q0, 0),
                  kStatBytes, bar(kXFull + s));
        issued = t + 1;
      }
      if (*abort_flag) {
        // each wait has its own time limit (a wait that gives up must not end the ones after it)
        {
          volatile int na = 0;
          mbar_wait(bar(kFixedFull), 0, &na);
        }
        for (int t = max(0, issued - kStages); t < issued; ++t) {
          volatile int na = 0;
          mbar_wait(bar(kXFull + (t & 1)), (t >> 1) & 1, &na);
        }
      }
    }
  } else if (warp == kMmaWarp) {
    // -------------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      // S_1^T = K Q_1^T, S_2^T = K Q_2^T, dP^T = V dO^T of step t for the queries of group c
      auto issue_scores = [&](int t, int c) {
        const uint32_t st = sbase + kKvOffX + (t & 1) * kKvStage;
        const uint32_t ro = kChainCols * c * 128;  // the chain's first query row in the stream tiles
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t a_k = tmem + kTmA + 8 * kk;  // K, resident in TMEM
          const uint64_t a_v = desc_kmajor(sbase + kKvOffV, kFixedChunk, kk);
          const uint32_t acc = kk > 0 ? 1u : 0u;
          mma_bf16_ts(tmem + kTmS1 + kChainCols * c, a_k, desc_kmajor(st + ro, kStreamChunk, kk), kIdescS, acc);
          mma_bf16_ts(tmem + kTmS2 + kChainCols * c, a_k, desc_kmajor(st + kStreamTile + ro, kStreamChunk, kk), kIdescS, acc);
          mma_bf16_ss(tmem + kTmDP + kChainCols * c, a_v, desc_kmajor(st + 2 * kStreamTile + ro, kStreamChunk, kk), kIdescS,
                      acc);
        }
        tc_commit(bar(kSFull + c));
      };
      // Issue order: scores(0); then per step t and group c: [wait P_c(t)] dV, dK of group c;
      // scores(t+1, c). Scores of step t+1 for group c overwrite only group c's columns, which
      // the accumulations just issued read first (MMAs execute in issue order), so each group
      // runs its own chain and the chains interleave on the tensor core.
      bool ok = mbar_wait(bar(kFixedFull), 0, abort_flag) && mbar_wait(bar(kAReady), 0, abort_flag) &&
                mbar_wait(bar(kXFull), 0, abort_flag);
      if (ok) {
        tc_fence_after();
        for (int c = 0; c < kChains; ++c) issue_scores(0, c);
      }
      for (int t = 0; ok && t < n_steps; ++t) {
        const int s = t & 1;
        const uint32_t st = sbase + kKvOffX + s * kKvStage;
        const uint32_t sQ1 = st, sQ2 = st + kStreamTile, sO = st + 2 * kStreamTile;
        const bool next = t + 1 < n_steps;
        // dV += W^T dO, dK += dS_1^T Q_1 + dS_2^T Q_2 (bf16 operands written over the scores)
#pragma unroll
        for (int c = 0; c < kChains; ++c) {
          if (!(ok = mbar_wait(bar(kPReady + c), t & 1, abort_flag))) break;
          tc_fence_after();
#pragma unroll
          for (int k2 = 0; k2 < kChainCols / 16; ++k2) {
            const int row = kChainCols * c + 16 * k2;                 // queries of this K-step
            const uint32_t col = operand_col(row);                    // their bf16 operands
            const uint32_t first = (t == 0 && c == 0 && k2 == 0) ? 0u : 1u;
            mma_bf16_ts(tmem + kTmAcc0, tmem + kTmS1 + col, desc_mnmajor(sO, kStreamChunk, row), kIdescAcc, first);
            mma_bf16_ts(tmem + kTmAcc1, tmem + kTmS2 + col, desc_mnmajor(sQ1, kStreamChunk, row), kIdescAcc, first);
            mma_bf16_ts(tmem + kTmAcc1, tmem + kTmDP + col, desc_mnmajor(sQ2, kStreamChunk, row), kIdescAcc, 1u);
          }
          if (next) {
            if (c == 0 && !(ok = mbar_wait(bar(kXFull + (s ^ 1)), ((t + 1) >> 1) & 1, abort_flag))) break;
            tc_fence_after();
            issue_scores(t + 1, c);
          }
        }
        if (!ok) break;
        tc_commit(bar(kXEmpty + s));
      }
      if (ok) tc_commit(bar(kDFull));
      tc_commit(bar(kDrain));
      volatile int no_abort = 0;
      mbar_wait(bar(kDrain), 0, &no_abort);
    }
  } else {
    // ------------------------------------------------------------------ elementwise
    const int cg = warp >> 2;                 // column group: queries kCols*cg .. of each step
    const int col0 = kCols * cg;
    const int r = 32 * (warp & 3) + lane;     // key row of the tile == TMEM lane
    const int key = k0 + r;
    const uint32_t trow = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    // K into TMEM for the score MMAs
    bool ok = __all_sync(0xffffffffu, mbar_wait(bar(kFixedFull), 0, abort_flag));
    if (ok) {
      tile_to_tmem(sbase + kKvOffK, trow, r, cg);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(kAReady));
    }
    for (int t = 0; ok && t < n_steps; ++t) {
      const int s = t & 1;
      const int q0 = (q_first + t % steps_per_pair) * 64;
      ok = __all_sync(0xffffffffu, mbar_wait(bar(kSFull + cg / kGroupsPerChain), t & 1, abort_flag));
      // the stage's stat records came by bulk copy: observe its completion directly (the
      // stage is refilled only after this step's operands have been consumed)
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar(kXFull + s), (t >> 1) & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      uint32_t s1[kCols], s2[kCols], dp[kCols];
      ld_cols(trow + kTmS1 + col0, s1);
      ld_cols(trow + kTmS2 + col0, s2);
      ld_cols(trow + kTmDP + col0, dp);
      ld_cols_wait(s1);
      ld_cols_wait(s2);
      ld_cols_wait(dp);
      // this group's columns of the five row-term arrays (shared, filled by bulk copy)
      const uint32_t rec = sbase + kKvOffX + s * kKvStage + 3 * kStreamTile + 4 * col0;
      // causal: only the two query blocks that overlap the key tile hold keys past a query;
      // window: blocks whose last query is window or more past the tile's first key hold
      // pairs outside the window
      const bool diag = p.causal && q0 < k0 + 128;
      const bool wedge = kWindow && q0 + 63 - k0 >= p.window;
      const int qbase = q0 + col0;
      const uint64_t sc2 = f2_pack(p.scale_log2, p.scale_log2);
      uint32_t w_pk[kCols / 2], d1_pk[kCols / 2], d2_pk[kCols / 2];
#pragma unroll
      for (int c4 = 0; c4 < kCols; c4 += 4) {
        uint64_t nl1[2], nl2[2], ne1[2], ne2[2], nlam[2];
        lds_f32x4(rec + 0 * 256 + 4 * c4, nl1[0], nl1[1]);
        lds_f32x4(rec + 1 * 256 + 4 * c4, nl2[0], nl2[1]);
        lds_f32x4(rec + 2 * 256 + 4 * c4, ne1[0], ne1[1]);
        lds_f32x4(rec + 3 * 256 + 4 * c4, ne2[0], ne2[1]);
        lds_f32x4(rec + 4 * 256 + 4 * c4, nlam[0], nlam[1]);
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          const int c = c4 + 2 * h2;  // columns c, c+1
          const uint64_t a1 = f2_fma(f2_pack(__uint_as_float(s1[c]), __uint_as_float(s1[c + 1])), sc2, nl1[h2]);
          const uint64_t a2 = f2_fma(f2_pack(__uint_as_float(s2[c]), __uint_as_float(s2[c + 1])), sc2, nl2[h2]);
          float x0, x1, y0, y1;
          f2_unpack(a1, x0, x1);
          f2_unpack(a2, y0, y1);
          float p10 = fast_exp2(x0), p11 = fast_exp2(x1), p20 = fast_exp2(y0), p21 = fast_exp2(y1);
          if (diag) {
            if (key > qbase + c) p10 = p20 = 0.f;
            if (key > qbase + c + 1) p11 = p21 = 0.f;
          }
          if (kWindow && wedge) {
            if (qbase + c - key >= p.window) p10 = p20 = 0.f;
            if (qbase + c + 1 - key >= p.window) p11 = p21 = 0.f;
          }
          const uint64_t P1 = f2_pack(p10, p11), P2 = f2_pack(p20, p21);
          const uint64_t dpp = f2_pack(__uint_as_float(dp[c]), __uint_as_float(dp[c + 1]));
          const uint64_t w = f2_fma(nlam[h2], P2, P1);                           // P1 - lambda P2
          const uint64_t d1 = f2_mul(P1, f2_add(dpp, ne1[h2]));                  // P1 (dP - E1)
          const uint64_t d2 = f2_mul(f2_mul(nlam[h2], P2), f2_add(dpp, ne2[h2]));  // -lambda P2 (dP - E2)
          float u0, u1;
          f2_unpack(w, u0, u1);
          w_pk[c >> 1] = pack_bf16x2(u0, u1);
          f2_unpack(d1, u0, u1);
          d1_pk[c >> 1] = pack_bf16x2(u0, u1);
          f2_unpack(d2, u0, u1);
          d2_pk[c >> 1] = pack_bf16x2(u0, u1);
        }
      }
      st_packed(trow + kTmS1 + col0, w_pk);
      st_packed(trow + kTmS2 + col0, d1_pk);
      st_packed(trow + kTmDP + col0, d2_pk);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(kPReady + cg / kGroupsPerChain));
    }
    if (ok) ok = mbar_wait(bar(kDFull), 0, abort_flag);
    if (__all_sync(0xffffffffu, ok && !*abort_flag)) {
      tc_fence_after();
      const int d0 = (128 / kGroups) * cg;
      const size_t off = ((row_base + (key < S ? key : 0)) * p.Hkv + g) * HD + d0;
      // rows of the whole launch: B x S, or the packed sequences' total
      const size_t total_rows = kVarlen ? static_cast<size_t>(__ldg(p.cu_seqlens + p.B)) : static_cast<size_t>(p.B) * p.S;
      const bool valid = key < S && checked(off + 128 / kGroups <= total_rows * p.Hkv * HD, p.err);
      store_row(trow + kTmAcc0 + d0, p.dv + off, 1.f, valid);
      store_row(trow + kTmAcc1 + d0, p.dk + off, p.scale, valid);
    }
  }
  teardown(tmem, abort_flag, p.err, warp);
}

// --------------------------------------------------------------------------------- dQ
template <bool kVarlen, bool kWindow>
__global__ void __launch_bounds__(kThreads, 1)
dq_sm100(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmO,
         const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + kQOffBar;
  auto bar = [&](int i) -> uint32_t { return bar0 + 8u * static_cast<uint32_t>(i); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kQOffBar + 128);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kQOffBar + 136);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_pairs = p.Hq >> 1, group = p.Hq / p.Hkv;
  const int pair = static_cast<int>(blockIdx.x) % n_pairs;
  const int b = static_cast<int>(blockIdx.x) / n_pairs;
  const int g = (2 * pair) / group;
  const int tile = p.causal ? p.n_tiles - 1 - static_cast<int>(blockIdx.y) : static_cast<int>(blockIdx.y);
  const int m0 = tile * 128;
  // sequence extent, as in the dK/dV kernel
  int S = p.S, tok0 = 0, tb = b, srow0 = 0;
  size_t sb = static_cast<size_t>(b) * n_pairs;
  if (kVarlen) {
    tok0 = __ldg(p.cu_seqlens + b);
    S = __ldg(p.cu_seqlens + b + 1) - tok0;
    tb = 0;
    sb = 0;
    srow0 = __ldg(p.pad_off + b);
  }
  if (m0 >= S) return;  // uniform over the CTA: the row tile lies past the sequence's end
  const size_t row_base = kVarlen ? static_cast<size_t>(tok0) : static_cast<size_t>(b) * p.S;
  const int nk = (S + 63) / 64;
  // key blocks kb_first .. kb_first+n_steps-1 (64 keys each); with a window the rows
  // m0 .. m0+127 see keys from m0-window+1 on
  const int kb_first = kWindow ? max(0, m0 - p.window + 1) / 64 : 0;
  const int n_steps = (p.causal ? min(nk, (m0 + 128) / 64) : nk) - kb_first;

  const uint32_t tmem = setup(bar0, tmem_slot, abort_flag, warp);

  if (warp == kProducerWarp) {
    if (lane == 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_arrive_expect_tx(bar(kFixedFull), 3 * kFixedTile);
      for (int c = 0; c < 2; ++c) {
        tma_load_4d(sbase + kQOffQ1 + c * kFixedChunk, &tmQ, bar(kFixedFull), c * 64, 2 * pair, tok0 + m0, tb);
        tma_load_4d(sbase + kQOffQ2 + c * kFixedChunk, &tmQ, bar(kFixedFull), c * 64, 2 * pair + 1, tok0 + m0, tb);
        tma_load_4d(sbase + kQOffO + c * kFixedChunk, &tmO, bar(kFixedFull), c * 64, pair, tok0 + m0, tb);
      }
      int issued = 0;
      for (int t = 0; t < n_steps; ++t) {
        const int s = t & 1;
        if (!mbar_wait(bar(kXEmpty + s), ((t >> 1) & 1) ^ 1, abort_flag)) break;
        const uint32_t st = sbase + kQOffX + s * kQStage;
        mbar_arrive_expect_tx(bar(kXFull + s), 2 * kStreamTile);
        for (int c = 0; c < 2; ++c) {
          tma_load_4d(st + c * kStreamChunk, &tmK, bar(kXFull + s), c * 64, g, tok0 + 64 * (kb_first + t), tb);
          tma_load_4d(st + kStreamTile + c * kStreamChunk, &tmV, bar(kXFull + s), c * 64, g,
                      tok0 + 64 * (kb_first + t), tb);
        }
        issued = t + 1;
      }
      if (*abort_flag) {
        // each wait has its own time limit (a wait that gives up must not end the ones after it)
        {
          volatile int na = 0;
          mbar_wait(bar(kFixedFull), 0, &na);
        }
        for (int t = max(0, issued - kStages); t < issued; ++t) {
          volatile int na = 0;
          mbar_wait(bar(kXFull + (t & 1)), (t >> 1) & 1, &na);
        }
      }
    }
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      // S_1 = Q_1 K^T, S_2 = Q_2 K^T, dP = dO V^T of key block t, keys 32h .. 32h+31
      auto issue_scores = [&](int t, int c) {
        const uint32_t sK = sbase + kQOffX + (t & 1) * kQStage, sV = sK + kStreamTile;
        const uint32_t ro = kChainCols * c * 128;  // the chain's first key row in the stream tiles
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint64_t b_k = desc_kmajor(sK + ro, kStreamChunk, kk);
          const uint32_t acc = kk > 0 ? 1u : 0u;
          mma_bf16_ts(tmem + kTmS1 + kChainCols * c, tmem + kTmA + 8 * kk, b_k, kIdescS, acc);  // Q_1 resident in TMEM
          mma_bf16_ss(tmem + kTmS2 + kChainCols * c, desc_kmajor(sbase + kQOffQ2, kFixedChunk, kk), b_k, kIdescS, acc);
          mma_bf16_ss(tmem + kTmDP + kChainCols * c, desc_kmajor(sbase + kQOffO, kFixedChunk, kk),
                      desc_kmajor(sV + ro, kStreamChunk, kk), kIdescS, acc);
        }
        tc_commit(bar(kSFull + c));
      };
      // same issue order as the dK/dV kernel
      bool ok = mbar_wait(bar(kFixedFull), 0, abort_flag) && mbar_wait(bar(kAReady), 0, abort_flag) &&
                mbar_wait(bar(kXFull), 0, abort_flag);
      if (ok) {
        tc_fence_after();
        for (int c = 0; c < kChains; ++c) issue_scores(0, c);
      }
      for (int t = 0; ok && t < n_steps; ++t) {
        const int s = t & 1;
        const uint32_t sK = sbase + kQOffX + s * kQStage;
        const bool next = t + 1 < n_steps;
        // dQ_1 += dS_1 K, dQ_2 += dS_2 K
#pragma unroll
        for (int c = 0; c < kChains; ++c) {
          if (!(ok = mbar_wait(bar(kPReady + c), t & 1, abort_flag))) break;
          tc_fence_after();
#pragma unroll
          for (int k2 = 0; k2 < kChainCols / 16; ++k2) {
            const int row = kChainCols * c + 16 * k2;                 // keys of this K-step
            const uint32_t col = operand_col(row);                    // their bf16 operands
            const uint32_t first = (t == 0 && c == 0 && k2 == 0) ? 0u : 1u;
            const uint64_t b_k = desc_mnmajor(sK, kStreamChunk, row);
            mma_bf16_ts(tmem + kTmAcc0, tmem + kTmS1 + col, b_k, kIdescAcc, first);
            mma_bf16_ts(tmem + kTmAcc1, tmem + kTmS2 + col, b_k, kIdescAcc, first);
          }
          if (next) {
            if (c == 0 && !(ok = mbar_wait(bar(kXFull + (s ^ 1)), ((t + 1) >> 1) & 1, abort_flag))) break;
            tc_fence_after();
            issue_scores(t + 1, c);
          }
        }
        if (!ok) break;
        tc_commit(bar(kXEmpty + s));
      }
      if (ok) tc_commit(bar(kDFull));
      tc_commit(bar(kDrain));
      volatile int no_abort = 0;
      mbar_wait(bar(kDrain), 0, &no_abort);
    }
  } else {
    const int cg = warp >> 2;                 // column group: keys kCols*cg .. of each step
    const int col0 = kCols * cg;
    const int r = 32 * (warp & 3) + lane;     // query row of the tile == TMEM lane
    const int qi = m0 + r;
    const uint32_t trow = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    // Q_1 into TMEM for the score MMAs
    bool ok = __all_sync(0xffffffffu, mbar_wait(bar(kFixedFull), 0, abort_flag));
    if (ok) {
      tile_to_tmem(sbase + kQOffQ1, trow, r, cg);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(kAReady));
    }
    // this row's terms (rows past S carry -lse = -inf: probabilities 0)
    const size_t bp = sb + pair;
    const int sr = srow0 + qi;  // this row in the row terms (past the sequence: -lse = -inf)
    const float nl1 = __ldg(p.stats + stat_index(bp, p.S_pad, sr, 0));
    const float nl2 = __ldg(p.stats + stat_index(bp, p.S_pad, sr, 1));
    const uint64_t ne1 = f2_pack(__ldg(p.stats + stat_index(bp, p.S_pad, sr, 2)), __ldg(p.stats + stat_index(bp, p.S_pad, sr, 2)));
    const uint64_t ne2 = f2_pack(__ldg(p.stats + stat_index(bp, p.S_pad, sr, 3)), __ldg(p.stats + stat_index(bp, p.S_pad, sr, 3)));
    const float nlam_s = __ldg(p.stats + stat_index(bp, p.S_pad, sr, 4));
    const uint64_t nl1_2 = f2_pack(nl1, nl1), nl2_2 = f2_pack(nl2, nl2), nlam = f2_pack(nlam_s, nlam_s);
    const uint64_t sc2 = f2_pack(p.scale_log2, p.scale_log2);
    for (int t = 0; ok && t < n_steps; ++t) {
      ok = __all_sync(0xffffffffu, mbar_wait(bar(kSFull + cg / kGroupsPerChain), t & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      uint32_t s1[kCols], s2[kCols], dp[kCols];
      ld_cols(trow + kTmS1 + col0, s1);
      ld_cols(trow + kTmS2 + col0, s2);
      ld_cols(trow + kTmDP + col0, dp);
      ld_cols_wait(s1);
      ld_cols_wait(s2);
      ld_cols_wait(dp);
      const int kb = kb_first + t;  // key block (t drives the stages and barriers)
      const int kbase = 64 * kb + col0;
      // tile-uniform: keys past the query (causal diagonal) or past S (ragged last block);
      // keys before some row's window start (the window's lower edge)
      const bool masked = (p.causal && 64 * kb + 63 > m0) || (64 * kb + 64 > S);
      const bool wedge = kWindow && 64 * kb < m0 + 128 - p.window;
      const int lim = p.causal ? min(qi, S - 1) : S - 1;  // last key this row sees
      const int lo = qi - p.window + 1;                      // first key it sees with a window
      uint32_t d1_pk[kCols / 2], d2_pk[kCols / 2];
#pragma unroll
      for (int c = 0; c < kCols; c += 2) {
        const uint64_t a1 = f2_fma(f2_pack(__uint_as_float(s1[c]), __uint_as_float(s1[c + 1])), sc2, nl1_2);
        const uint64_t a2 = f2_fma(f2_pack(__uint_as_float(s2[c]), __uint_as_float(s2[c + 1])), sc2, nl2_2);
        float x0, x1, y0, y1;
        f2_unpack(a1, x0, x1);
        f2_unpack(a2, y0, y1);
        float p10 = fast_exp2(x0), p11 = fast_exp2(x1), p20 = fast_exp2(y0), p21 = fast_exp2(y1);
        if (masked) {
          if (kbase + c > lim) p10 = p20 = 0.f;
          if (kbase + c + 1 > lim) p11 = p21 = 0.f;
        }
        if (kWindow && wedge) {
          if (kbase + c < lo) p10 = p20 = 0.f;
          if (kbase + c + 1 < lo) p11 = p21 = 0.f;
        }
        const uint64_t dpp = f2_pack(__uint_as_float(dp[c]), __uint_as_float(dp[c + 1]));
        const uint64_t d1 = f2_mul(f2_pack(p10, p11), f2_add(dpp, ne1));
        const uint64_t d2 = f2_mul(f2_mul(nlam, f2_pack(p20, p21)), f2_add(dpp, ne2));
        float u0, u1;
        f2_unpack(d1, u0, u1);
        d1_pk[c >> 1] = pack_bf16x2(u0, u1);
        f2_unpack(d2, u0, u1);
        d2_pk[c >> 1] = pack_bf16x2(u0, u1);
      }
      st_packed(trow + kTmS1 + col0, d1_pk);
      st_packed(trow + kTmS2 + col0, d2_pk);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(kPReady + cg / kGroupsPerChain));
    }
    if (ok) ok = mbar_wait(bar(kDFull), 0, abort_flag);
    if (__all_sync(0xffffffffu, ok && !*abort_flag)) {
      tc_fence_after();
      const int d0 = (128 / kGroups) * cg;
      const size_t off = ((row_base + (qi < S ? qi : 0)) * p.Hq + 2 * pair) * HD + d0;
      const size_t total_rows = kVarlen ? static_cast<size_t>(__ldg(p.cu_seqlens + p.B)) : static_cast<size_t>(p.B) * p.S;
      const bool valid = qi < S && checked(off + HD + 128 / kGroups <= total_rows * p.Hq * HD, p.err);
      store_row(trow + kTmAcc0 + d0, p.dq + off, p.scale, valid);
      store_row(trow + kTmAcc1 + d0, p.dq + off + HD, p.scale, valid);
    }
  }
  teardown(tmem, abort_flag, p.err, warp);
}

}  // namespace bwd_tc

size_t backward_stats_bytes(int B, int S, int Hq) {
  const size_t s_pad = (static_cast<size_t>(S) + bwd_tc::kRowPad - 1) / bwd_tc::kRowPad * bwd_tc::kRowPad;
  return static_cast<size_t>(B) * (Hq / 2) * s_pad * bwd_tc::kStatArrays * sizeof(float);
}

// Packed sequences: rows of the row terms for T tokens in B sequences, each padded to 128.
static size_t varlen_stat_rows(int B, int T) {
  return (static_cast<size_t>(T) + static_cast<size_t>(bwd_tc::kRowPad) * B + bwd_tc::kRowPad - 1) /
         bwd_tc::kRowPad * bwd_tc::kRowPad;
}

size_t backward_varlen_workspace_bytes(int B, int T, int Hq) {
  const size_t stats = static_cast<size_t>(Hq / 2) * varlen_stat_rows(B, T) * bwd_tc::kStatArrays * sizeof(float);
  return stats + (static_cast<size_t>(B) + 1 + 3) / 4 * 16;  // + the B+1 padded offsets
}

cudaError_t launch_backward_sm100(const CUtensorMap& tmQ64, const CUtensorMap& tmQ128, const CUtensorMap& tmO64,
                                  const CUtensorMap& tmO128, const CUtensorMap& tmK64, const CUtensorMap& tmK128,
                                  const CUtensorMap& tmV64, const CUtensorMap& tmV128, const float* lambda,
                                  const __nv_bfloat16* o_branch, const float* lse, const __nv_bfloat16* dout,
                                  __nv_bfloat16* dq, __nv_bfloat16* dk, __nv_bfloat16* dv, float* dlambda,
                                  float* workspace, int* err, int B, int S, int Hq, int Hkv, int causal,
                                  cudaStream_t stream, const int32_t* cu_seqlens, int total_tokens, int window) {
  using namespace bwd_tc;
  const int n_pairs = Hq / 2;
  Params p;
  cudaError_t e;
  if (cu_seqlens) {
    // S is the longest sequence; the row terms of all sequences form one padded batch
    const int S_pad = static_cast<int>(varlen_stat_rows(B, total_tokens));
    int* pad_off = reinterpret_cast<int*>(workspace + static_cast<size_t>(n_pairs) * S_pad * kStatArrays);
    pad_offsets_kernel<<<1, 32, 0, stream>>>(cu_seqlens, pad_off, B);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const long long warps = static_cast<long long>(S_pad) * n_pairs;
    preprocess_varlen_kernel<<<static_cast<unsigned>((warps + 3) / 4), 128, 0, stream>>>(
        dout, o_branch, lse, lambda, workspace, dlambda, cu_seqlens, pad_off, B, S_pad, n_pairs);
    p.S_pad = S_pad;
    p.pad_off = pad_off;
  } else {
    const int S_pad = (S + kRowPad - 1) / kRowPad * kRowPad;
    const long long warps = static_cast<long long>(B) * S_pad * n_pairs;
    preprocess_kernel<<<static_cast<unsigned>((warps + 3) / 4), 128, 0, stream>>>(dout, o_branch, lse, lambda,
                                                                                    workspace, dlambda, B, S, S_pad,
                                                                                    n_pairs);
    p.S_pad = S_pad;
    p.pad_off = nullptr;
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  p.stats = workspace;
  p.dq = dq;
  p.dk = dk;
  p.dv = dv;
  p.err = err;
  p.B = B;
  p.S = S;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.causal = causal;
  p.window = window;
  p.cu_seqlens = cu_seqlens;
  p.n_tiles = (S + 127) / 128;
  p.scale = 1.f / sqrtf(static_cast<float>(HD));
  p.scale_log2 = 1.4426950408889634f * p.scale;
  auto run = [&](auto kdkdv, auto kdq) {
    cudaError_t r = cudaFuncSetAttribute(kdkdv, cudaFuncAttributeMaxDynamicSharedMemorySize, kKvSmem);
    if (r != cudaSuccess) return r;
    r = cudaFuncSetAttribute(kdq, cudaFuncAttributeMaxDynamicSharedMemorySize, kQSmem);
    if (r != cudaSuccess) return r;
    kdkdv<<<dim3(B * Hkv, p.n_tiles), kThreads, kKvSmem, stream>>>(tmQ64, tmO64, tmK128, tmV128, p);
    r = cudaGetLastError();
    if (r != cudaSuccess) return r;
    kdq<<<dim3(B * n_pairs, p.n_tiles), kThreads, kQSmem, stream>>>(tmQ128, tmO128, tmK64, tmV64, p);
    return cudaGetLastError();
  };
  if (cu_seqlens && window > 0) return run(dkdv_sm100<true, true>, dq_sm100<true, true>);
  if (cu_seqlens) return run(dkdv_sm100<true, false>, dq_sm100<true, false>);
  if (window > 0) return run(dkdv_sm100<false, true>, dq_sm100<false, true>);
  return run(dkdv_sm100<false, false>, dq_sm100<false, false>);
}

}  // namespace da2
