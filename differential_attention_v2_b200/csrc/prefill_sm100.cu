// prefill_sm100.cu -- bf16 DiffAttn V2 prefill on the 5th-generation tensor cores (sm_100a).
//
// Operator ("Differential Attention (V2)" lesson, "The differential concept"; causal mask of
// the "Attention variants" lesson, Step 1; V2 pairing of "Differential Transformer V2 soll
// KI-Training stabiler machen", shared-KV section):
//   out[b,i,p] = softmax(q[b,i,2p] K_g^T/sqrt(D)) V_g - lambda[b,i,p] softmax(q[b,i,2p+1] K_g^T/sqrt(D)) V_g
//
// A work item is a 128-row query tile of one pair (both heads) of one batch element. The
// kernel is persistent: one CTA per SM walks its share of the items, ranked heaviest first
// (last row tile first) and dealt out to the CTAs in snake order, so the next item's Q and
// K/V loads and its first score GEMMs overlap the previous item's last softmax and its
// epilogue. Packed sequences deal out only their non-empty items (see work_item). Each 128x128 K and V tile of the shared KV head is brought into shared memory by
// TMA ONCE and feeds both heads. The four GEMM blocks per KV tile run on tcgen05 with fp32
// accumulators in tensor memory:
//
//   TMEM columns   [  0,128) S1 = Q1 K^T   (P1, bf16, is written over its first 64 columns)
//                  [128,256) S2 = Q2 K^T   (P2 likewise)
//                  [256,384) O1 += P1 V
//                  [384,512) O2 += P2 V
//
// Warp roles (384 threads):
//   warps 0-3  softmax of branch 1 (head 2p): thread r owns query row r of the tile
//   warps 4-7  softmax of branch 2 (head 2p+1)
//   warp 8     TMA producer (Q per item, K/V tiles through a 2-stage ring across items)
//   warp 9     tcgen05 MMA issuer; also allocates and frees tensor memory
//   warps 10-11 idle: they complete warpgroup 2, which hands its registers to warps 0-7;
//              in the fused-lambda form they compute each item's V2 lambda (see below)
//
// Issue order on the tensor core for KV tile j: S1_j, PV2_{j-1}, S2_j, PV1_j. Softmax of
// branch 1 on S1_j overlaps PV2_{j-1} and S2_j; softmax of branch 2 on S2_j overlaps PV1_j
// and S1_{j+1}. tcgen05.mma instructions from one thread execute in issue order, so S_b(j+1)
// overwrites the P_b(j) columns only after PV_b(j) has read them.
//
// Online softmax per branch in the log2 domain: x = s * log2(e)/sqrt(D), P = 2^(x - m).
// The running max m is raised only when a row's max exceeds it by more than 8 (a factor of
// 256); then O and l are rescaled by 2^(m_old - m_new). O/l is the same for any such m, so
// this is exact up to rounding while skipping most rescales. The epilogue forms
// O1/l1 - lambda O2/l2 in fp32 and rounds once to bf16.
//
// Fused-lambda form (kLamFused, [B,S] inputs): lambda is not read from memory but computed
// in the kernel from the tokens' hidden states x and the projection of "Differential
// Transformer V2 soll KI-Training stabiler machen" ("Weniger Ausreisser und
// Gradientenspitzen": lambda per token and head, bounded by a sigmoid):
// lambda[t, p] = sigmoid(x[t] . w[p] + bias[p]). Warps 10 and 11 take 64 rows each of every
// item's tile, dot products over d_model on the CUDA cores, and hand the 128 values to the
// epilogue through a two-slot ring in shared memory.

#include <cstdlib>

#include "bounds.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace da2 {
namespace prefill {

constexpr int BM = 128;  // query rows per CTA
constexpr int BN = 128;  // keys per KV tile
constexpr int HD = 128;  // head dim
constexpr int kThreads = 384;
// Register split (setmaxnreg, per warpgroup): the kernel launches with kRegsLaunch per thread;
// warpgroup 2 (producer, MMA issuer, two idle warps) gives registers back so the two softmax
// warpgroups can hold a row's 128 scores and its packed P without spilling. The shares add up
// to no more than the launch total (128 * 96 + 256 * 200 = 63,488 <= 384 * 168 = 64,512; per SM
// sub-partition, whose warps are w, w+4, w+8: (200 + 200 + 96) * 32 <= 16,384). ptxas compiles
// each role's code to its share: at 200 the softmax path has no spills (at 168 it spilled).
constexpr int kRegsLaunch = 168, kRegsSmall = 96, kRegsSoftmax = 200;
static_assert(128 * kRegsSmall + 256 * kRegsSoftmax <= kThreads * kRegsLaunch, "register split exceeds the launch");

constexpr uint32_t kChunkBytes = 128 * 64 * 2;     // 128 rows x 64 bf16 (one swizzle-128B half)
constexpr uint32_t kTileBytes = 2 * kChunkBytes;   // 128 rows x 128 bf16

// Shared-memory plan of the two kernel forms. One CTA per item: K and V tiles of 128 keys x
// 128 d in a 2-stage ring. CTA pair (two CTAs of a cluster on an SM pair share every MMA):
// each CTA holds half of every K tile (64 keys x 128 d) and half of every V tile (128 keys x
// 64 d), in a 4-stage ring. Both use 192 KB before the barriers.
template <bool kPair>
struct Ring {
  static constexpr int kStages = kPair ? 4 : 2;
  static constexpr uint32_t kKChunk = kPair ? 64 * 64 * 2 : kChunkBytes;  // one 64-d half of a K stage
  static constexpr uint32_t kKStage = 2 * kKChunk;
  static constexpr uint32_t kVStage = kPair ? kChunkBytes : kTileBytes;
};

constexpr uint32_t kOffQ = 0;                                         // Q1, Q2
constexpr uint32_t kOffK = kOffQ + 2 * kTileBytes;                    // K stages
constexpr uint32_t kOffBar = kOffK + 2 * 2 * kTileBytes;              // after the K and V stages
static_assert(kOffK + Ring<false>::kStages * (Ring<false>::kKStage + Ring<false>::kVStage) == kOffBar, "smem plan");
static_assert(kOffK + Ring<true>::kStages * (Ring<true>::kKStage + Ring<true>::kVStage) == kOffBar, "smem plan");
template <bool kPair>
__host__ __device__ constexpr uint32_t off_v() { return kOffK + Ring<kPair>::kStages * Ring<kPair>::kKStage; }
constexpr uint32_t kOffMisc = kOffBar + 256;                  // tmem slot, abort flag
constexpr uint32_t kOffL = kOffMisc + 64;                     // [item parity][branch][row] fp32 row sums
// packed sequences: sequence ids sorted by row-tile count (longest first), then the counts;
// in the fused-lambda form (never with packed sequences) the same bytes hold the lambda ring
constexpr int kMaxSortedSeqs = 256;
constexpr uint32_t kOffSeq = kOffL + 2 * 2 * BM * 4;
constexpr uint32_t kOffLamRing = kOffSeq;                      // [slot][row] fp32
static_assert(2 * BM * 4 <= 2 * kMaxSortedSeqs * 4, "lambda ring");
// out staging for the tensor stores: 32 rows x 32 columns of bf16 per softmax warp
constexpr uint32_t kStageBytes = 32 * 32 * 2;
constexpr uint32_t kOffStage = (kOffSeq + 2 * kMaxSortedSeqs * 4 + 1023) / 1024 * 1024;
constexpr uint32_t kSmemUsed = kOffStage + 8 * kStageBytes;
constexpr uint32_t kSmemBytes = kSmemUsed + 1024;             // slack for 1024-B alignment
static_assert(kSmemBytes <= 227 * 1024, "shared memory of one CTA");

// mbarrier slots (8 bytes each)
enum Bar : int {
  kQFull = 0,
  kKFull = 1,    // +stage
  kKEmpty = 5,   // +stage
  kVFull = 9,    // +stage
  kVEmpty = 13,  // +stage
  kSFull = 17,   // +branch
  kPFull = 19,   // +2*branch+half: P of keys 64*half .. 64*half+63 is in TMEM
  kOFull = 23,
  kDrain = 24,
  kQEmpty = 25,  // the item's last score GEMM has read Q
  kOEmpty = 26,  // every softmax thread has read O1, O2 of the item into registers
  kLx = 27,      // both branches' row sums of the item are in shared memory
  kLamFull = 28,   // +slot: the fused lambda of the slot's item is in shared memory
  kLamEmpty = 30,  // +slot: every softmax thread has read it
  kNumBars = 32
};
static_assert(kNumBars * 8 <= 256, "barrier slots");

constexpr uint32_t kTmS1 = 0, kTmS2 = 128, kTmO1 = 256, kTmO2 = 384;

struct Params {
  const float* lambda;    // [B,S,Hq/2]
  __nv_bfloat16* out;     // [B,S,Hq/2,D]
  __nv_bfloat16* o_branch;  // training forward: [B,S,Hq,D] per-head normalised O_b (null = inference)
  float* lse;             // training forward: [B,S,Hq] log2-domain log-sum-exp of the scaled scores
  int* err;               // device error word
  int B, S, Hq, Hkv, causal;
  int window;             // causal sliding window (keys i-window+1 .. i); 0 = none
  const int* cu_seqlens;  // packed sequences: sequence b is tokens cu[b] .. cu[b+1]-1; null = [B,S]
  int n_row_tiles;
  int n_items;            // B * (Hq/2) * n_row_tiles
  int sorted_seqs;        // packed sequences dealt as a dense list of non-empty items (B <= kMaxSortedSeqs)
  float scale_log2;       // log2(e)/sqrt(D)
  // fused lambda (kLamFused): lambda[t, p] = sigmoid(x[t] . wt[p] + bias[p])
  const __nv_bfloat16* lam_x;   // [B*S, d_model] token hidden states
  const __nv_bfloat16* lam_wt;  // [Hq/2, d_model] projection, one row per pair
  const float* lam_bias;        // [Hq/2] or null
  float* lam_out;               // [B*S, Hq/2] fp32 copy of the computed lambda, or null
  int d_model;                  // a multiple of 8
};

// One work item: query rows m0 .. m0+127 of pair `pair` of sequence b, visiting KV tiles
// j_first .. j_first+n_kv-1 (n_kv = 0: the tile lies past the end of a packed sequence).
struct WorkItem {
  int b, pair, tile, m0;
  int S, tok0, tb;        // sequence length; its first row and batch index in the tensor maps
  int j_first, n_kv;
  size_t row_base;        // first output row of the sequence
};

// Walk over the dense list of non-empty packed-sequence items: rank r holds row tile
// t = n_row_tiles-1-r of the n_seq longest sequences (those with more than t row tiles, a
// prefix of the sorted list), pair fastest; base is the list index of the rank's first item.
struct SortedCursor {
  int r = 0, base = 0, n_seq = 0;
};

// The k-th item of this CTA; false once they are exhausted. Items are ranked by row tile,
// last tile first (causal work grows with the tile index), and band k of gridDim.x items goes
// to the CTAs in ascending order for even k and descending order for odd k. With sorted
// packed sequences only non-empty items are listed (seq_id, seq_nt: sorted ids and row-tile
// counts; n_dense: the list's length); a role's item indices only grow, so its cursor only
// moves forward.
// With kPair the unit of work is a pair of pairs of one KV head: cluster c takes the item and
// its CTA of rank r computes pair 2u + r (u = the unit's index among the Hq/4 units).
template <bool kVarlen, bool kWindow, bool kPair>
__device__ __forceinline__ bool work_item(const Params& p, int k, WorkItem& w, SortedCursor& cur,
                                          const int* seq_id, const int* seq_nt, int n_dense, uint32_t cta_rank) {
  constexpr int kCtas = kPair ? 2 : 1;
  const int n_ctas = static_cast<int>(gridDim.x) / kCtas;   // CTAs, or clusters of two
  const int c = static_cast<int>(blockIdx.x) / kCtas;
  const int idx = k * n_ctas + ((k & 1) ? n_ctas - 1 - c : c);
  const int n_pairs = p.Hq >> (kPair ? 2 : 1);   // work units per (sequence, row tile)
  if (kVarlen && p.sorted_seqs) {
    if (idx >= n_dense) return false;
    int t = p.n_row_tiles - 1 - cur.r;
    while (true) {
      if (t < 0) return false;  // unreachable: the ranks hold exactly n_dense items
      while (cur.n_seq < p.B && seq_nt[cur.n_seq] > t) ++cur.n_seq;
      const int n_rank = cur.n_seq * n_pairs;
      if (idx < cur.base + n_rank) break;
      cur.base += n_rank;
      ++cur.r;
      --t;
    }
    const int within = idx - cur.base;
    const int si = within / n_pairs;
    w.tile = t;
    w.b = seq_id[si];
    w.pair = within - si * n_pairs;
  } else {
    if (idx >= p.n_items) return false;  // only in the last band; later bands are empty too
    const int per_tile = p.B * n_pairs;
    const int rank = idx / per_tile;
    const int bp = idx - rank * per_tile;
    w.tile = p.n_row_tiles - 1 - rank;
    w.b = bp / n_pairs;
    w.pair = bp - w.b * n_pairs;
  }
  if (kPair) w.pair = 2 * w.pair + static_cast<int>(cta_rank);
  w.m0 = w.tile * BM;
  w.S = p.S;
  w.tok0 = 0;
  w.tb = w.b;
  if (kVarlen) {
    w.tok0 = __ldg(p.cu_seqlens + w.b);
    w.S = __ldg(p.cu_seqlens + w.b + 1) - w.tok0;
    w.tb = 0;
  }
  w.row_base = kVarlen ? static_cast<size_t>(w.tok0) : static_cast<size_t>(w.b) * p.S;
  if (w.m0 >= w.S) {
    w.j_first = 0;
    w.n_kv = 0;
    return true;
  }
  const int n_kv_total = (w.S + BN - 1) / BN;
  const int j_last = p.causal ? min(w.tile, n_kv_total - 1) : n_kv_total - 1;
  // with a sliding window the first KV tile holds key m0 - window + 1 (or key 0)
  const int win_lo = w.m0 - p.window + 1;
  w.j_first = (kWindow && win_lo > 0) ? win_lo / BN : 0;
  w.n_kv = j_last - w.j_first + 1;
  return true;
}

// Set scores of keys outside columns lo..hi of this thread's NC x 32 columns to -inf.
template <int NC>
__device__ __forceinline__ void mask_row(uint32_t (&sr)[NC][32], int lo, int hi) {
#pragma unroll
  for (int c = 0; c < NC; ++c)
#pragma unroll
    for (int e = 0; e < 32; ++e)
      if (32 * c + e > hi || 32 * c + e < lo) sr[c][e] = __float_as_uint(-INFINITY);
}

// Max of this thread's NC x 32 raw scores: 3-input max, four independent chains.
template <int NC>
__device__ __forceinline__ float row_max(const uint32_t (&sr)[NC][32]) {
  float m0 = -INFINITY, m1 = -INFINITY, m2 = -INFINITY, m3 = -INFINITY;
#pragma unroll
  for (int c = 0; c < NC; ++c)
#pragma unroll
    for (int e = 0; e < 32; e += 8) {
      m0 = fmax3(m0, __uint_as_float(sr[c][e + 0]), __uint_as_float(sr[c][e + 1]));
      m1 = fmax3(m1, __uint_as_float(sr[c][e + 2]), __uint_as_float(sr[c][e + 3]));
      m2 = fmax3(m2, __uint_as_float(sr[c][e + 4]), __uint_as_float(sr[c][e + 5]));
      m3 = fmax3(m3, __uint_as_float(sr[c][e + 6]), __uint_as_float(sr[c][e + 7]));
    }
  return fmax3(m0, m1, fmaxf(m2, m3));
}

// 2^x of two values on the FMA pipe (no MUFU): x = n + f with n = rint(x) and f in
// [-1/2, 1/2]; 2^f by a cubic fitted for minimax relative error on [-1/2, 1/2] (Remez
// exchange, max relative error 7.5e-5, well under bf16's 2^-9); 2^n is added to the
// exponent field. x is clamped to -126 so the exponent never underflows past zero.
// Adding 1.5 * 2^23 rounds x to an integer held in the low mantissa bits of t, so
// bits(t) << 23 == n << 23 (mod 2^32).
constexpr float kExpShift = 12582912.0f;  // 1.5 * 2^23
constexpr float kExpC0 = 0.99992806f, kExpC1 = 0.69326097f, kExpC2 = 0.24261113f, kExpC3 = 0.05517167f;

__device__ __forceinline__ void exp2_poly_x2(float x0, float x1, float& y0, float& y1) {
  const uint64_t x = f2_pack(fmaxf(x0, -126.f), fmaxf(x1, -126.f));
  const uint64_t t = f2_add(x, f2_pack(kExpShift, kExpShift));
  const uint64_t n = f2_add(t, f2_pack(-kExpShift, -kExpShift));
  const uint64_t f = f2_fma(n, f2_pack(-1.f, -1.f), x);
  uint64_t q = f2_fma(f2_pack(kExpC3, kExpC3), f, f2_pack(kExpC2, kExpC2));
  q = f2_fma(q, f, f2_pack(kExpC1, kExpC1));
  q = f2_fma(q, f, f2_pack(kExpC0, kExpC0));
  float q0, q1, t0, t1;
  f2_unpack(q, q0, q1);
  f2_unpack(t, t0, t1);
  y0 = __int_as_float(__float_as_int(q0) + (__float_as_int(t0) << 23));
  y1 = __int_as_float(__float_as_int(q1) + (__float_as_int(t1) << 23));
}

// Pairs of keys whose exponentials go to the FMA pipe instead of the MUFU: one pair in
// kExpFmaEvery (0: none). Measured on B200 (B=4 x 4k and 1 x 32k causal): none is fastest.
// The kernel runs at the 1 kW power cap, where the extra FMA-pipe work lowers the SM clock
// by more than the MUFU time it saves.
#ifndef DA2_EXP_FMA_EVERY
#define DA2_EXP_FMA_EVERY 0
#endif
constexpr int kExpFmaEvery = DA2_EXP_FMA_EVERY;
__host__ __device__ constexpr bool exp_on_fma(int pair) {
  return kExpFmaEvery > 0 && (pair % (kExpFmaEvery > 0 ? kExpFmaEvery : 1)) == (kExpFmaEvery - 1);
}

// P = 2^(s*scale - m) for keys 64*half .. 64*half+63 of the row, packed to bf16 pairs and
// stored over TMEM columns 32*half .. 32*half+31 of the row's S tile (keys 2c, 2c+1 ->
// column c). Returns the fp32 sum of these P. The exponent argument of two keys is one
// packed FMA; with kEmulate, one pair in four is exponentiated on the FMA pipe.
template <bool kEmulate>
__device__ __forceinline__ float exp_pack_store(const uint32_t (&sr)[4][32], int half, float scale, float m_use,
                                                uint32_t taddr) {
  const uint64_t scale2 = f2_pack(scale, scale);
  const uint64_t negm2 = f2_pack(-m_use, -m_use);
  uint64_t sum_a = f2_pack(0.f, 0.f), sum_b = f2_pack(0.f, 0.f);
  uint32_t pk[32];
#pragma unroll
  for (int cc = 0; cc < 2; ++cc) {
    const int c = 2 * half + cc;
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
      const uint64_t arg = f2_fma(f2_pack(__uint_as_float(sr[c][e]), __uint_as_float(sr[c][e + 1])), scale2, negm2);
      float a0, a1, p0, p1;
      f2_unpack(arg, a0, a1);
      if (kEmulate && exp_on_fma(e >> 1)) {
        exp2_poly_x2(a0, a1, p0, p1);
      } else {
        p0 = fast_exp2(a0);
        p1 = fast_exp2(a1);
      }
      if ((e >> 1) & 1)
        sum_b = f2_add(sum_b, f2_pack(p0, p1));
      else
        sum_a = f2_add(sum_a, f2_pack(p0, p1));
      pk[cc * 16 + (e >> 1)] = pack_bf16x2(p0, p1);
    }
  }
  tmem_st_32x32b_x32(taddr + 32 * half, pk);
  float s0, s1, s2, s3;
  f2_unpack(sum_a, s0, s1);
  f2_unpack(sum_b, s2, s3);
  return (s0 + s1) + (s2 + s3);
}

// 16 bytes of a stream read once (not kept in L1).
__device__ __forceinline__ uint4 ld_stream_v4(const void* ptr) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(ptr));
  return v;
}

// acc (two fp32 partial sums) += the dot product of 8 bf16 values a and w (bf16 -> fp32 is
// exact: the 16 bits move to the top of the word).
__device__ __forceinline__ uint64_t dot8_bf16(uint4 a, uint4 w, uint64_t acc) {
  const uint32_t av[4] = {a.x, a.y, a.z, a.w}, wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint64_t x2 = f2_pack(__uint_as_float(av[i] << 16), __uint_as_float(av[i] & 0xFFFF0000u));
    const uint64_t w2 = f2_pack(__uint_as_float(wv[i] << 16), __uint_as_float(wv[i] & 0xFFFF0000u));
    acc = f2_fma(x2, w2, acc);
  }
  return acc;
}

// 32 bf16 values (16 packed pairs) of one row to global memory: two 256-bit stores where dst
// is 32-byte aligned (the caller's buffers need only 16), else four 128-bit ones.
__device__ __forceinline__ void store_row32(__nv_bfloat16* dst, const uint32_t (&v)[16]) {
  if ((reinterpret_cast<uintptr_t>(dst) & 31u) == 0) {
    st_global_v8(dst, v);
    st_global_v8(dst + 16, v + 8);
  } else {
    uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
    for (int i = 0; i < 4; ++i) d[i] = make_uint4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
  }
}

// Waits on barriers that the other CTA arrives on use the default (CTA-scope acquire) form,
// as the arrivals do; what they order is tensor memory, through the tcgen05 fences.
constexpr bool kClusterAcquire = false;

// A bounded wait on one of this CTA's barriers (pwait), or, by the MMA thread, on a barrier
// that the other CTA's threads arrive on (pwait_x: acquire at cluster scope). With kPair a wait
// that gives up also raises the other CTA's abort flag (flag_addr: this CTA's flag).
template <bool kPair>
__device__ __forceinline__ void raise_peer_abort(uint32_t flag_addr) {
  if constexpr (kPair) st_cluster_u32(mapa_shared(flag_addr, cluster_ctarank() ^ 1u), 1u);
}
template <bool kPair>
__device__ __forceinline__ bool pwait(uint32_t b, uint32_t parity, volatile int* abort_flag, uint32_t flag_addr) {
  const bool r = mbar_wait(b, parity, abort_flag);
  if (kPair && !r) raise_peer_abort<kPair>(flag_addr);
  return r;
}
template <bool kPair>
__device__ __forceinline__ bool pwait_x(uint32_t b, uint32_t parity, volatile int* abort_flag, uint32_t flag_addr) {
  const bool r = (kPair && kClusterAcquire) ? mbar_wait_cluster(b, parity, abort_flag) : mbar_wait(b, parity, abort_flag);
  if (kPair && !r) raise_peer_abort<kPair>(flag_addr);
  return r;
}

// A softmax thread's arrival on a barrier the MMA thread waits on, after its tensor-memory
// stores or loads: every thread on this CTA's barrier, or with kPair once per warp on the even
// CTA's barrier (bar: this CTA's copy).
template <bool kPair>
__device__ __forceinline__ void arrive_for_mma(uint32_t bar, int lane) {
  tc_fence_before();
  if constexpr (kPair) {
    __syncwarp();
    if (lane == 0) mbar_arrive_cluster(mapa_shared(bar, 0));
  } else {
    mbar_arrive(bar);
  }
}

// kVarlen: packed sequences (p.cu_seqlens); kWindow: causal sliding window (p.window). The
// plain [B,S] prefill is the <false, false, *> instance and carries neither.
// kPair: a cluster of two CTAs on an SM pair computes two pairs of the same KV head over the
// same 128 query rows. The even CTA's MMA thread issues every GEMM once for both
// (tcgen05.mma.cta_group::2, M = 256: each CTA's own 128 rows of Q or P against a shared K or
// V tile of which each CTA loaded half), so per unit of work the tensor-core instructions and
// the shared-memory operand reads per SM are cut (A 4 KB + half of B 2 KB per score
// instruction and SM instead of 4 + 4 KB) and each SM loads half of every K/V tile.
// Protocol across the pair (all loads are plain per-CTA TMA copies, none multicast):
//   * copies of both CTAs count their bytes on the even CTA's full barriers (the even CTA's
//     producer announces both halves' bytes);
//   * the MMA thread's commits arrive on the barrier at the same offset in both CTAs
//     (S ready, O ready, K/V/Q stage free);
//   * each softmax warp of either CTA arrives once on the even CTA's P and O-read barriers;
//   * a wait that gives up raises the abort flag of both CTAs; both CTAs leave through one
//     cluster barrier, after every copy and commit addressed to them has landed.
template <bool kVarlen, bool kWindow, bool kPair, bool kLamFused = false>
__global__ void __launch_bounds__(kThreads, 1)
diffattn_prefill_sm100(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmKh,
                       const __grid_constant__ CUtensorMap tmO, const Params p) {
  using R = Ring<kPair>;
  constexpr int kStages = R::kStages;
  constexpr uint32_t kOffV = off_v<kPair>();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  auto bar = [&](int i) -> uint32_t { return sbase + kOffBar + 8u * static_cast<uint32_t>(i); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 8);
  float* l_xchg = reinterpret_cast<float*>(smem + kOffL);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_pairs = p.Hq >> 1;
  const int group = p.Hq / p.Hkv;
  const uint32_t cta_rank = kPair ? cluster_ctarank() : 0u;
  const bool leader = cta_rank == 0;
  // the even CTA's copy of barrier i in the cluster's shared window (this CTA's own without
  // kPair); computed where used, so that no register holds it across the loops
  auto bar_lead = [&](int i) -> uint32_t { return kPair ? mapa_shared(bar(i), 0) : bar(i); };
  const uint32_t flag_addr = sbase + kOffMisc + 8;  // the abort flag's shared address

  int* seq_id = reinterpret_cast<int*>(smem + kOffSeq);
  int* seq_nt = seq_id + kMaxSortedSeqs;
  int* n_dense_slot = reinterpret_cast<int*>(smem + kOffMisc + 16);
  if (threadIdx.x == 0) {
    for (int i = 0; i < kNumBars; ++i) {
      uint32_t count = 1;
      // P and O-read barriers: every softmax thread of the branch / CTA, or with kPair one
      // arrival per softmax warp of both CTAs
      if (i >= kPFull && i < kPFull + 4) count = kPair ? 8 : 128;
      if (i == kOEmpty) count = kPair ? 16 : 256;
      if (i == kLx) count = 256;
      if (i == kLamFull || i == kLamFull + 1) count = 64;
      if (i == kLamEmpty || i == kLamEmpty + 1) count = 256;
      mbar_init(bar(i), count);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (kVarlen && p.sorted_seqs) {
    // Sequences by row-tile count, longest first (ties by index). Counts are clamped to
    // [0, n_row_tiles]: rows past the longest length the caller declared are not computed,
    // as in the one-CTA-per-item launch. The row-sum array is free until the first epilogue
    // and holds the counts meanwhile.
    int* nt = reinterpret_cast<int*>(l_xchg);
    for (int b = threadIdx.x; b < p.B; b += kThreads) {
      const int len = __ldg(p.cu_seqlens + b + 1) - __ldg(p.cu_seqlens + b);
      nt[b] = min(max((len + BM - 1) / BM, 0), p.n_row_tiles);
    }
    __syncthreads();
    for (int b = threadIdx.x; b < p.B; b += kThreads) {
      const int nb = nt[b];
      int rank = 0;
      for (int b2 = 0; b2 < p.B; ++b2) rank += (nt[b2] > nb || (nt[b2] == nb && b2 < b)) ? 1 : 0;
      if (checked(rank < kMaxSortedSeqs, p.err)) {
        seq_id[rank] = b;
        seq_nt[rank] = nb;
      }
    }
    if (threadIdx.x == 0) {
      int total = 0;
      for (int b = 0; b < p.B; ++b) total += nt[b];
      *n_dense_slot = total * (p.Hq >> (kPair ? 2 : 1));
    }
  }
  if (warp == 8 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(kPair ? &tmKh : &tmK);
    tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmO);
  }
  if (warp == 9) {
    if constexpr (kPair) {
      tmem_alloc_pair(smem_u32(tmem_slot), 512);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_u32(tmem_slot), 512);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (kPair) cluster_sync();  // both CTAs' barriers and tensor memory exist
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int n_dense = (kVarlen && p.sorted_seqs) ? *n_dense_slot : 0;
  WorkItem w;
  SortedCursor cur;

  if (warp >= 8) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsSmall));
    if (warp == 8) {
      // ------------------------------------------------------------------ TMA producer
      if (lane == 0) {
        // Counts over all items of this CTA: KV tiles (ring stage and phase) and Q tiles.
        int k_issued = 0, v_issued = 0, q_issued = 0;
        bool ok = true;
        // the even CTA announces the bytes of both CTAs' halves
        const uint32_t pair_mult = kPair ? 2u : 1u;
        for (int k = 0; ok && work_item<kVarlen, kWindow, kPair>(p, k, w, cur, seq_id, seq_nt, n_dense, cta_rank);
             ++k) {
          if (w.n_kv == 0) continue;
          // the single Q buffer is free once the previous item's last score GEMM has read it
          if (q_issued > 0 && !(ok = pwait<kPair>(bar(kQEmpty), (q_issued - 1) & 1, abort_flag, flag_addr))) break;
          if (leader) mbar_arrive_expect_tx(bar(kQFull), pair_mult * 2 * kTileBytes);
          for (int h = 0; h < 2; ++h)
            for (int c = 0; c < 2; ++c) {
              const uint32_t dst = sbase + kOffQ + h * kTileBytes + c * kChunkBytes;
              if (!checked(within(dst, kChunkBytes, sbase + kOffQ, 2 * kTileBytes) && 2 * w.pair + h < p.Hq, p.err))
                continue;
              if constexpr (kPair)
                tma_load_4d_pair(dst, &tmQ, bar_lead(kQFull), c * 64, 2 * w.pair + h, w.tok0 + w.m0, w.tb);
              else
                tma_load_4d(dst, &tmQ, bar(kQFull), c * 64, 2 * w.pair + h, w.tok0 + w.m0, w.tb);
            }
          ++q_issued;
          const int g = (2 * w.pair) / group;
          for (int it = 0; it < w.n_kv; ++it) {
            const int j = w.j_first + it;
            const int n = k_issued;  // this CTA's KV tile count so far
            const int s = n % kStages;
            const uint32_t ph = (n / kStages) & 1;
            if (!(ok = pwait<kPair>(bar(kKEmpty + s), ph ^ 1, abort_flag, flag_addr))) break;
            if (leader) mbar_arrive_expect_tx(bar(kKFull + s), pair_mult * R::kKStage);
            for (int c = 0; c < 2; ++c) {
              const uint32_t dst = sbase + kOffK + s * R::kKStage + c * R::kKChunk;
              if (!checked(within(dst, R::kKChunk, sbase + kOffK, kStages * R::kKStage) && g < p.Hkv, p.err)) continue;
              if constexpr (kPair)  // keys 64*rank .. 64*rank+63 of the tile, all 128 d
                tma_load_4d_pair(dst, &tmKh, bar_lead(kKFull + s), c * 64, g, w.tok0 + j * BN + 64 * cta_rank, w.tb);
              else
                tma_load_4d(dst, &tmK, bar(kKFull + s), c * 64, g, w.tok0 + j * BN, w.tb);
            }
            k_issued = n + 1;
            if (!(ok = pwait<kPair>(bar(kVEmpty + s), ph ^ 1, abort_flag, flag_addr))) break;
            if (leader) mbar_arrive_expect_tx(bar(kVFull + s), pair_mult * R::kVStage);
            if (!checked(within(sbase + kOffV + s * R::kVStage, R::kVStage, sbase + kOffV, kStages * R::kVStage) &&
                             g < p.Hkv, p.err)) {
              // skipped: the stage's barrier stays short and the MMA thread's wait gives up
            } else if constexpr (kPair) {  // all 128 keys, d 64*rank .. 64*rank+63
              tma_load_4d_pair(sbase + kOffV + s * R::kVStage, &tmV, bar_lead(kVFull + s), 64 * cta_rank, g,
                               w.tok0 + j * BN, w.tb);
            } else {
              for (int c = 0; c < 2; ++c)
                tma_load_4d(sbase + kOffV + s * R::kVStage + c * kChunkBytes, &tmV, bar(kVFull + s), c * 64, g,
                            w.tok0 + j * BN, w.tb);
            }
            v_issued = n + 1;
          }
        }
        if (*abort_flag) {
          if constexpr (kPair) {
            // the copies' completions count on the even CTA's barriers, which this CTA may not
            // be able to see complete: give any copy still in flight time to land
            const uint64_t t0 = global_timer_ns();
            while (global_timer_ns() - t0 < 2000000ull) __nanosleep(1000);
          } else {
            // let copies still in flight land before the CTA's shared memory is released: at
            // most one Q tile and one K and one V tile per stage can be outstanding. Each wait
            // has its own time limit (a wait that gives up must not end the ones after it).
            if (q_issued > 0) {
              volatile int na = 0;
              mbar_wait(bar(kQFull), (q_issued - 1) & 1, &na);
            }
            for (int n = max(0, k_issued - kStages); n < k_issued; ++n) {
              volatile int na = 0;
              mbar_wait(bar(kKFull + n % kStages), (n / kStages) & 1, &na);
            }
            for (int n = max(0, v_issued - kStages); n < v_issued; ++n) {
              volatile int na = 0;
              mbar_wait(bar(kVFull + n % kStages), (n / kStages) & 1, &na);
            }
          }
        } else if (kPair) {
          // the even CTA's last commits (stage and Q releases) arrive on this CTA's barriers:
          // take them before the CTA can leave (an abort raised meanwhile ends the waits; the
          // even CTA then drains its MMAs, and with them these commits, before both leave)
          for (int n = max(0, k_issued - kStages); n < k_issued; ++n)
            mbar_wait(bar(kKEmpty + n % kStages), (n / kStages) & 1, abort_flag);
          for (int n = max(0, v_issued - kStages); n < v_issued; ++n)
            mbar_wait(bar(kVEmpty + n % kStages), (n / kStages) & 1, abort_flag);
          if (q_issued > 0) mbar_wait(bar(kQEmpty), (q_issued - 1) & 1, abort_flag);
        }
      }
    } else if (warp == 9) {
      // -------------------------------------------------------------------- MMA issuer
      // (with kPair only the even CTA's thread issues, for both CTAs)
      if (lane == 0 && leader) {
        constexpr int kM = kPair ? 2 * BM : BM;
        constexpr uint32_t idesc_qk = idesc_bf16_f32(kM, BN, false);
        constexpr uint32_t idesc_pv = idesc_bf16_f32(kM, HD, true);
        auto desc_q = [&](int h, int kk) {
          return sdesc_sw128(sbase + kOffQ + h * kTileBytes + (kk >> 2) * kChunkBytes + (kk & 3) * 32, 16, 1024);
        };
        // K stage: keys x d with d contiguous (K-major B operand); with kPair each CTA holds 64 keys
        auto desc_k = [&](int s, int kk) {
          return sdesc_sw128(sbase + kOffK + s * R::kKStage + (kk >> 2) * R::kKChunk + (kk & 3) * 32, 16, 1024);
        };
        // V stage: keys x d with d contiguous (MN-major B operand); 16 keys per K-step; with
        // kPair each CTA holds one 64-wide half of d (the leading offset is then unused)
        auto desc_v = [&](int s, int kk) {
          return sdesc_sw128(sbase + kOffV + s * R::kVStage + kk * 2048, kChunkBytes, 1024);
        };
        auto mma_ss = [&](uint32_t d, uint64_t a, uint64_t b, uint32_t id, uint32_t acc) {
          if constexpr (kPair) mma_bf16_ss_pair(d, a, b, id, acc);
          else mma_bf16_ss(d, a, b, id, acc);
        };
        auto commit = [&](int i) {
          if constexpr (kPair) tc_commit_pair(bar(i), 0x3);
          else tc_commit(bar(i));
        };
        // O_b (+)= P_b V for this CTA's KV tile number n (ring stage n % kStages, P barrier
        // phase n & 1): the first 64 keys as soon as that half of P is in TMEM, the other 64
        // when the second half is. acc = false starts the item's sum.
        auto issue_pv = [&](uint32_t o_tmem, uint32_t p_tmem, int n, bool acc, uint32_t half0, uint32_t half1) {
  #pragma unroll
          for (int h = 0; h < 2; ++h) {
            if (!pwait_x<kPair>(h ? half1 : half0, n & 1, abort_flag, flag_addr)) return false;
            tc_fence_after();
  #pragma unroll
            for (int kk = 4 * h; kk < 4 * h + 4; ++kk) {
              const uint32_t acc_kk = (acc || kk > 0) ? 1u : 0u;
              if constexpr (kPair) mma_bf16_ts_pair(o_tmem, p_tmem + kk * 8, desc_v(n % kStages, kk), idesc_pv, acc_kk);
              else mma_bf16_ts(o_tmem, p_tmem + kk * 8, desc_v(n % kStages, kk), idesc_pv, acc_kk);
            }
          }
          return true;
        };
        int n0 = 0;       // KV tiles of earlier items
        int n_items = 0;  // items done
        // the four 128-column accumulators fill the 512 allocated columns from column 0
        bool ok = checked((tmem & 0xFFFFu) == 0u && kTmO2 + HD <= 512u, p.err);
        for (int k = 0; ok && work_item<kVarlen, kWindow, kPair>(p, k, w, cur, seq_id, seq_nt, n_dense, cta_rank);
             ++k) {
          if (w.n_kv == 0) continue;
          if (!(ok = pwait<kPair>(bar(kQFull), n_items & 1, abort_flag, flag_addr))) break;
          for (int j = 0; j < w.n_kv; ++j) {
            const int n = n0 + j;
            const int s = n % kStages;
            const uint32_t ph = (n / kStages) & 1;
            if (!(ok = pwait<kPair>(bar(kKFull + s), ph, abort_flag, flag_addr))) break;
            tc_fence_after();
  #pragma unroll
            for (int kk = 0; kk < HD / 16; ++kk)
              mma_ss(tmem + kTmS1, desc_q(0, kk), desc_k(s, kk), idesc_qk, kk > 0 ? 1u : 0u);
            commit(kSFull + 0);
            if (j > 0) {
              if (!(ok = issue_pv(tmem + kTmO2, tmem + kTmS2, n - 1, j > 1, bar(kPFull + 2), bar(kPFull + 3)))) break;
              commit(kVEmpty + (n - 1) % kStages);
            }
  #pragma unroll
            for (int kk = 0; kk < HD / 16; ++kk)
              mma_ss(tmem + kTmS2, desc_q(1, kk), desc_k(s, kk), idesc_qk, kk > 0 ? 1u : 0u);
            commit(kSFull + 1);
            commit(kKEmpty + s);
            if (j == w.n_kv - 1) commit(kQEmpty);
            if (!(ok = pwait<kPair>(bar(kVFull + s), ph, abort_flag, flag_addr))) break;
            if (j == 0 && n_items > 0) {
              // the first PV of an item overwrites O1 (and O2 after it): the previous item's
              // epilogue must have read them
              if (!(ok = pwait_x<kPair>(bar(kOEmpty), (n_items - 1) & 1, abort_flag, flag_addr))) break;
              tc_fence_after();
            }
            if (!(ok = issue_pv(tmem + kTmO1, tmem + kTmS1, n, j > 0, bar(kPFull + 0), bar(kPFull + 1)))) break;
          }
          if (!ok) break;
          const int nl = n0 + w.n_kv - 1;
          if (!(ok = issue_pv(tmem + kTmO2, tmem + kTmS2, nl, w.n_kv > 1, bar(kPFull + 2), bar(kPFull + 3)))) break;
          commit(kVEmpty + nl % kStages);
          commit(kOFull);
          n0 += w.n_kv;
          ++n_items;
        }
        // every MMA of this CTA (with kPair: of both CTAs) must be complete before tensor
        // memory is freed
        if constexpr (kPair) tc_commit_pair_local(bar(kDrain));
        else tc_commit(bar(kDrain));
        volatile int no_abort = 0;
        mbar_wait(bar(kDrain), 0, &no_abort);
      }
    } else if constexpr (kLamFused) {
      // ------------------------------------------- fused V2 lambda (warps 10 and 11)
      // Warp 10 takes rows 0-63 of each item's tile, warp 11 rows 64-127, two rows at a time;
      // lane l sums elements 8l .. 8l+7 of every 256 of d_model, then the warp adds the lanes.
      float* lam_ring = reinterpret_cast<float*>(smem + kOffLamRing);
      const int row0 = (warp - 10) * 64;
      const int n_pairs_l = p.Hq >> 1;
      int n_li = 0;  // items with KV tiles so far (the ring's count, as the softmax warps')
      bool ok = true;
      for (int k = 0; ok && work_item<kVarlen, kWindow, kPair>(p, k, w, cur, seq_id, seq_nt, n_dense, cta_rank);
           ++k) {
        if (w.n_kv == 0) continue;
        const int s = n_li & 1;
        ok = __all_sync(0xffffffffu, mbar_wait(bar(kLamEmpty + s), ((n_li >> 1) & 1) ^ 1, abort_flag));
        if (!ok) break;
        const __nv_bfloat16* wrow = p.lam_wt + static_cast<size_t>(w.pair) * p.d_model;
        const float bias = p.lam_bias != nullptr ? __ldg(p.lam_bias + w.pair) : 0.f;
#pragma unroll 1
        for (int rr = 0; rr < 64; rr += 2) {
          const int qa = w.m0 + row0 + rr;  // rows qa and qa + 1 of the sequence
          const bool va = qa < w.S, vb = qa + 1 < w.S;
          const __nv_bfloat16* xa = p.lam_x + (w.row_base + (va ? qa : 0)) * p.d_model;
          const __nv_bfloat16* xb = p.lam_x + (w.row_base + (vb ? qa + 1 : 0)) * p.d_model;
          uint64_t acc_a = f2_pack(0.f, 0.f), acc_b = f2_pack(0.f, 0.f);
#pragma unroll 4
          for (int d = 8 * lane; d < p.d_model; d += 256) {
            const uint4 wv = __ldg(reinterpret_cast<const uint4*>(wrow + d));
            const uint4 av = va ? ld_stream_v4(xa + d) : make_uint4(0u, 0u, 0u, 0u);
            const uint4 bv = vb ? ld_stream_v4(xb + d) : make_uint4(0u, 0u, 0u, 0u);
            acc_a = dot8_bf16(av, wv, acc_a);
            acc_b = dot8_bf16(bv, wv, acc_b);
          }
          float a0, a1, b0, b1;
          f2_unpack(acc_a, a0, a1);
          f2_unpack(acc_b, b0, b1);
          float sa = a0 + a1, sb = b0 + b1;
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) {
            sa += __shfl_xor_sync(0xffffffffu, sa, o);
            sb += __shfl_xor_sync(0xffffffffu, sb, o);
          }
          if (lane == 0) {
            const float la = va ? 1.f / (1.f + expf(-(sa + bias))) : 0.f;
            const float lb = vb ? 1.f / (1.f + expf(-(sb + bias))) : 0.f;
            if (checked(s * BM + row0 + rr + 1 < 2 * BM, p.err)) {
              lam_ring[s * BM + row0 + rr] = la;
              lam_ring[s * BM + row0 + rr + 1] = lb;
            }
            if (p.lam_out != nullptr) {
              const size_t lam_elems = static_cast<size_t>(p.B) * p.S * n_pairs_l;
              const size_t ia = (w.row_base + qa) * n_pairs_l + w.pair;
              if (va && checked(ia < lam_elems, p.err)) p.lam_out[ia] = la;
              if (vb && checked(ia + n_pairs_l < lam_elems, p.err)) p.lam_out[ia + n_pairs_l] = lb;
            }
          }
        }
        mbar_arrive(bar(kLamFull + s));
        ++n_li;
      }
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
    const int br = warp >> 2;               // branch 0 (head 2p) or 1 (head 2p+1)
    const int r = threadIdx.x & 127;        // row of the tile == TMEM lane
    const uint32_t trow = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const uint32_t s_col = br ? kTmS2 : kTmS1;
    const uint32_t o_col = br ? kTmO2 : kTmO1;
    int n0 = 0;       // KV tiles of earlier items
    int n_items = 0;  // items done
    bool ok = true;

    for (int k = 0; ok && work_item<kVarlen, kWindow, kPair>(p, k, w, cur, seq_id, seq_nt, n_dense, cta_rank); ++k) {
      if (w.n_kv == 0) continue;
      const int qi = w.m0 + r;  // query index of this row within its sequence
      const int S = w.S;
      // this row's lambda, loaded at the start of the item so that its latency hides under
      // the item's tiles instead of lying on the epilogue's path
      const size_t lam_off = (w.row_base + (qi < S ? qi : 0)) * n_pairs + w.pair;
      bool lam_ok = qi < S;
      if constexpr (kDebugBounds) {
        const size_t rows = kVarlen ? static_cast<size_t>(__ldg(p.cu_seqlens + p.B)) : static_cast<size_t>(p.B) * p.S;
        lam_ok = lam_ok && checked(lam_off < rows * n_pairs, p.err);
      }
      float lam_row = (!kLamFused && lam_ok) ? __ldg(p.lambda + lam_off) : 0.f;
      float m_run = -INFINITY;
      float l_run = 0.f;
      for (int it = 0; it < w.n_kv; ++it) {
        const int j = w.j_first + it;  // KV tile index (key position); n0 + it drives the barriers
        ok = __all_sync(0xffffffffu, pwait<kPair>(bar(kSFull + br), (n0 + it) & 1, abort_flag, flag_addr));
        if (!ok) break;
        tc_fence_after();
        uint32_t sr[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld_32x32b_x32(trow + s_col + 32 * c, sr[c]);
        tmem_ld_wait(sr[0]);
        reg_fence(sr[1]);
        reg_fence(sr[2]);
        reg_fence(sr[3]);

        // Keys visible to this row in this tile are columns 0..lim; only the diagonal tile of
        // a causal launch and a ragged last key tile have lim < 127.
        // tile_masked is uniform over the CTA: every branch below that holds a warp-collective
        // tcgen05 instruction must be taken by all 32 lanes together
        // some row of the tile has keys of this KV tile below its window
        const bool win_edge = kWindow && j * BN < w.m0 + BM - p.window;
        const bool tile_masked = (p.causal && j == w.tile) || ((j + 1) * BN > S) || win_edge;
        // dead_h: no row of the warp sees a key of 64-key half h (the diagonal tile's upper
        // half for rows 0-63, a window's first tile's lower half for rows 64-127)
        bool dead0 = false, dead1 = false;
        if (tile_masked) {
          int hi = BN - 1;
          if (p.causal && j == w.tile) hi = r;
          hi = min(hi, S - 1 - j * BN);
          const int lo = kWindow ? qi - p.window + 1 - j * BN : 0;
          mask_row<4>(sr, lo, hi);
          dead0 = __all_sync(0xffffffffu, hi < 0 || lo > 63);
          dead1 = __all_sync(0xffffffffu, hi < 64 || lo > 127);
        }
        const float mx = row_max<4>(sr) * p.scale_log2;

        // raise the running max only when the tile's max exceeds it by more than 2^8
        const bool rescale = mx > m_run + 8.f;
        float alpha = 1.f;
        if (rescale) {
          alpha = fast_exp2(m_run - mx);  // 0 on the first tile
          l_run *= alpha;
          m_run = mx;
        }
        // the warp rescales its 32 rows together (alpha = 1 for rows that keep their max)
        if (__any_sync(0xffffffffu, rescale) && it > 0) {
          // O_b holds the sum up to the previous tile, complete: S_b(j) was committed after that
          // tile's PV_b,
          // and PV_b(j) is issued only after this thread arrives on the P barriers below
#pragma unroll 1
          for (int c = 0; c < 8; ++c) {
            uint32_t o[16];
            tmem_ld_32x32b_x16(trow + o_col + 16 * c, o);
            tmem_ld_wait16(o);
#pragma unroll
            for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            tmem_st_32x32b_x16(trow + o_col + 16 * c, o);
          }
        }
        const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
        float lsum = 0.f;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          // a half no row of the warp sees gets P = 0 without its exponentials (all 2^-inf =
          // 0); masked tiles take every other exponential on the MUFU so masked keys stay
          // exactly 0
          if (half ? dead1 : dead0) {
            uint32_t zero[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) zero[e] = 0u;
            tmem_st_32x32b_x32(trow + s_col + 32 * half, zero);
          } else {
            lsum += tile_masked ? exp_pack_store<false>(sr, half, p.scale_log2, m_use, trow + s_col)
                                : exp_pack_store<true>(sr, half, p.scale_log2, m_use, trow + s_col);
          }
          tmem_st_wait();
          arrive_for_mma<kPair>(bar(kPFull + 2 * br + half), lane);
        }
        l_run += lsum;
      }
      if (!ok) break;
      n0 += w.n_kv;
      if constexpr (kLamFused) {
        // this row's lambda from warps 10 and 11
        const int ls = n_items & 1;
        ok = __all_sync(0xffffffffu, pwait<kPair>(bar(kLamFull + ls), (n_items >> 1) & 1, abort_flag, flag_addr));
        if (!ok) break;
        lam_row = reinterpret_cast<const float*>(smem + kOffLamRing)[ls * BM + r];
        mbar_arrive(bar(kLamEmpty + ls));
      }

      // ---- epilogue of the item: out = O1/l1 - lambda O2/l2; thread r of branch br writes
      // columns 64*br .. 64*br+63 of row r, so the two branches swap row sums through shared
      // memory (one buffer per item parity: a buffer is rewritten two items later, after
      // every thread has passed the kLx and kOEmpty barriers of the item in between). The
      // row sums go out before the wait for O, and the first 32 of the thread's columns of O1
      // and O2 are requested from tensor memory before the wait for the other branch's sums,
      // so that the load's latency passes under that wait.
      float* lx = l_xchg + (n_items & 1) * 2 * BM;
      lx[br * BM + r] = l_run;
      // training forward: A_b = 2^(s * scale_log2 - lse) recomputes the probabilities later
      // rows of the whole launch: B x S, or the packed sequences' total
      const size_t total_rows = kVarlen ? static_cast<size_t>(__ldg(p.cu_seqlens + p.B)) : static_cast<size_t>(p.B) * p.S;
      if (p.lse != nullptr && qi < S &&
          checked((w.row_base + qi) * p.Hq + 2 * w.pair + br < total_rows * p.Hq, p.err))
        p.lse[(w.row_base + qi) * p.Hq + 2 * w.pair + br] = (m_run == -INFINITY ? 0.f : m_run) + __log2f(l_run);
      mbar_arrive(bar(kLx));
      ok = __all_sync(0xffffffffu, pwait<kPair>(bar(kOFull), n_items & 1, abort_flag, flag_addr));
      if (!ok) break;
      const uint32_t col0 = 64 * br;
      uint32_t o1[32], o2[32];
      tc_fence_after();
      tmem_ld_32x32b_x32(trow + kTmO1 + col0, o1);
      tmem_ld_32x32b_x32(trow + kTmO2 + col0, o2);
      ok = pwait<kPair>(bar(kLx), n_items & 1, abort_flag, flag_addr) && ok;
      tmem_ld_wait(o1);
      reg_fence(o2);
      ok = __all_sync(0xffffffffu, ok && !*abort_flag);
      if (!ok) break;
      {
        const float inv1 = 1.f / lx[r];
        const float inv2 = 1.f / lx[BM + r];
        const size_t row_off = (w.row_base + (qi < S ? qi : 0)) * n_pairs + w.pair;
        const bool row_valid = qi < S && checked(row_off < total_rows * n_pairs, p.err);
        const float lam = row_valid ? lam_row : 0.f;
        // out leaves through shared memory and one tensor store per warp and 32 columns
        // (rows of a [B,S] launch past S are clipped by the store; a packed sequence's rows
        // past its end belong to the next sequence, so a warp whose 32 rows reach past the
        // end stores its valid rows itself)
        const int slab = w.m0 + 32 * (warp & 3);
        const bool via_tma = kVarlen ? slab + 32 <= S : slab < S;
        const uint32_t stage = sbase + kOffStage + kStageBytes * static_cast<uint32_t>(warp);
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          const uint32_t col = col0 + 32 * cc;
          if (cc == 1) {
            tmem_ld_wait(o1);
            reg_fence(o2);
            // O1, O2 are read: the next item's first PV may overwrite them
            arrive_for_mma<kPair>(bar(kOEmpty), lane);
          }
          if (p.o_branch != nullptr && row_valid) {
            // per-head normalised O_1, O_2 of the pair, same columns as this thread's out slice
#pragma unroll
            for (int hb = 0; hb < 2; ++hb) {
              const uint32_t* o = hb ? o2 : o1;
              const float inv = hb ? inv2 : inv1;
              uint32_t ob[16];
#pragma unroll
              for (int e = 0; e < 16; ++e)
                ob[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * inv, __uint_as_float(o[2 * e + 1]) * inv);
              store_row32(p.o_branch + ((w.row_base + qi) * p.Hq + 2 * w.pair + hb) * HD + col, ob);
            }
          }
          uint32_t packed[16];
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            // each branch normalised with its own rounding, then one fused subtract: equal
            // branches (Q1 == Q2, lambda == 1) cancel exactly
            const float y0 =
                __fmaf_rn(-lam, __fmul_rn(__uint_as_float(o2[e]), inv2), __fmul_rn(__uint_as_float(o1[e]), inv1));
            const float y1 = __fmaf_rn(-lam, __fmul_rn(__uint_as_float(o2[e + 1]), inv2),
                                       __fmul_rn(__uint_as_float(o1[e + 1]), inv1));
            packed[e >> 1] = pack_bf16x2(y0, y1);
          }
          if (cc == 0) {
            tmem_ld_32x32b_x32(trow + kTmO1 + col0 + 32, o1);
            tmem_ld_32x32b_x32(trow + kTmO2 + col0 + 32, o2);
          }
          if (via_tma) {
            // the warp's buffer is free once its previous store has read it
            if (lane == 0) bulk_wait_read();
            __syncwarp();
            // row `lane` of the 32 x 32 box, 64-byte swizzle: 16-byte chunk c of row l sits
            // at chunk c ^ ((l >> 1) & 3) (8 consecutive rows then fill all 32 banks)
#pragma unroll
            for (int c = 0; c < 4; ++c)
              st_shared_v4(stage + 64u * lane + ((static_cast<uint32_t>(c) ^ ((lane >> 1) & 3u)) << 4),
                           packed[4 * c], packed[4 * c + 1], packed[4 * c + 2], packed[4 * c + 3]);
            fence_proxy_async_shared();
            __syncwarp();
            if (lane == 0) {
              tma_store_4d(&tmO, stage, static_cast<int>(col), w.pair, w.tok0 + slab, w.tb);
              bulk_commit();
            }
          } else if (row_valid) {
            store_row32(p.out + row_off * HD + col, packed);
          }
        }
      }
      ++n_items;
    }
    // every tensor store of this thread has completed before the CTA exits
    if (lane == 0) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  if constexpr (kPair) {
    // neither CTA leaves (or frees tensor memory) while the other may still address it: the
    // even CTA has drained every MMA, each producer has taken the commits addressed to it
    cluster_sync();
  }
  if (threadIdx.x == 0 && *abort_flag) atomicCAS(p.err, 0, kErrPrefillWait);
  if (warp == 9) {
    __syncwarp();  // lane 0 ran the MMA loop alone; dealloc is warp-collective
    tc_fence_after();
    if constexpr (kPair) tmem_dealloc_pair(tmem, 512);
    else tmem_dealloc(tmem, 512);
  }
}

}  // namespace prefill

cudaError_t launch_prefill(const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV,
                           const CUtensorMap* tmKh, const CUtensorMap& tmO, const float* lambda, __nv_bfloat16* out, int* err, int B, int S,
                           int Hq, int Hkv, int causal, int window, const int* cu_seqlens, cudaStream_t stream,
                           __nv_bfloat16* o_branch, float* lse) {
  using namespace prefill;
  Params p;
  p.lambda = lambda;
  p.out = out;
  p.o_branch = o_branch;
  p.lse = lse;
  p.err = err;
  p.B = B;
  p.S = S;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.causal = causal;
  p.window = window;
  p.cu_seqlens = cu_seqlens;  // with packed sequences S is the longest sequence's length
  p.n_row_tiles = (S + BM - 1) / BM;
  p.sorted_seqs = (cu_seqlens != nullptr && B <= kMaxSortedSeqs) ? 1 : 0;
  p.scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(HD));
  int device = 0, n_sms = 0;
  cudaError_t e = cudaGetDevice(&device);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&n_sms, cudaDevAttrMultiProcessorCount, device);
  if (e != cudaSuccess) return e;
  const bool one_per_item = cu_seqlens != nullptr && !p.sorted_seqs;

  // The CTA-pair form runs when DA2_PREFILL_CTA_PAIR=1 is set in the environment, every KV head
  // has an even number of pairs (GQA group a multiple of 4), the persistent deal applies and
  // the caller passed the half-tile K map. It gives bit-identical results; on B200 it measured
  // about 2% below the one-CTA form in short runs and the same under a sustained load (what
  // paces both is each branch's chain of softmax, PV and next score GEMM, and then the power
  // cap, not the number of MMA instructions or operand bytes), so one CTA per item is the
  // default.
  const int group = Hq / Hkv;
  const char* env = getenv("DA2_PREFILL_CTA_PAIR");
  const bool pair_wanted = env != nullptr && env[0] == '1';
  const bool use_pair = pair_wanted && tmKh != nullptr && (group % 4) == 0 && !one_per_item &&
                        !(cu_seqlens != nullptr && window > 0);
  if (use_pair) {
    p.n_items = B * (Hq / 4) * p.n_row_tiles;
    if (p.n_items == 0) return cudaSuccess;
    auto kernel = cu_seqlens ? diffattn_prefill_sm100<true, false, true>
                             : (window > 0 ? diffattn_prefill_sm100<false, true, true>
                                           : diffattn_prefill_sm100<false, false, true>);
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cfg.gridDim = dim3(static_cast<unsigned>(n_sms & ~1), 1, 1);
    // persistent: as many clusters as can be resident at once (an SM pair each)
    int n_clusters = 0;
    e = cudaOccupancyMaxActiveClusters(&n_clusters, kernel, &cfg);
    if (e != cudaSuccess) return e;
    if (n_clusters <= 0) return cudaErrorInvalidConfiguration;
    n_clusters = n_clusters < p.n_items ? n_clusters : p.n_items;
    cfg.gridDim = dim3(static_cast<unsigned>(2 * n_clusters), 1, 1);
    e = cudaLaunchKernelEx(&cfg, kernel, tmQ, tmK, tmV, *tmKh, tmO, p);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
  }

  p.n_items = B * (Hq / 2) * p.n_row_tiles;
  auto kernel = cu_seqlens ? (window > 0 ? diffattn_prefill_sm100<true, true, false>
                                         : diffattn_prefill_sm100<true, false, false>)
                           : (window > 0 ? diffattn_prefill_sm100<false, true, false>
                                         : diffattn_prefill_sm100<false, false, false>);
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  if (p.n_items == 0) return cudaSuccess;
  // Persistent: one CTA per SM (the shared memory admits one), each walking its items. Packed
  // sequences of mixed length leave many items empty (row tiles past a short sequence's end);
  // up to kMaxSortedSeqs sequences the CTAs deal out only the non-empty ones (p.sorted_seqs),
  // beyond that every item of the full grid gets its own CTA and the hardware's CTA scheduler
  // balances them (a static deal that includes the empty items measured 745 against 800
  // TFLOP/s for 8 sequences of 512-3584 tokens).
  const int n_ctas = (one_per_item || p.n_items < n_sms) ? p.n_items : n_sms;
  kernel<<<n_ctas, kThreads, kSmemBytes, stream>>>(tmQ, tmK, tmV, tmK, tmO, p);
  return cudaGetLastError();
}

cudaError_t launch_prefill_lambda_fused(const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV,
                                        const CUtensorMap& tmO, const __nv_bfloat16* x, const __nv_bfloat16* w_t,
                                        const float* bias, float* lambda_out, int d_model, __nv_bfloat16* out,
                                        int* err, int B, int S, int Hq, int Hkv, int causal, cudaStream_t stream) {
  using namespace prefill;
  Params p{};
  p.lambda = nullptr;
  p.out = out;
  p.err = err;
  p.B = B;
  p.S = S;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.causal = causal;
  p.window = 0;
  p.cu_seqlens = nullptr;
  p.n_row_tiles = (S + BM - 1) / BM;
  p.sorted_seqs = 0;
  p.scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(HD));
  p.lam_x = x;
  p.lam_wt = w_t;
  p.lam_bias = bias;
  p.lam_out = lambda_out;
  p.d_model = d_model;
  p.n_items = B * (Hq / 2) * p.n_row_tiles;
  int device = 0, n_sms = 0;
  cudaError_t e = cudaGetDevice(&device);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&n_sms, cudaDevAttrMultiProcessorCount, device);
  if (e != cudaSuccess) return e;
  auto kernel = diffattn_prefill_sm100<false, false, false, true>;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  if (p.n_items == 0) return cudaSuccess;
  const int n_ctas = p.n_items < n_sms ? p.n_items : n_sms;
  kernel<<<n_ctas, kThreads, kSmemBytes, stream>>>(tmQ, tmK, tmV, tmK, tmO, p);
  return cudaGetLastError();
}

}  // namespace da2
