// decode_noalloc.cu -- the bf16 decode step for callers that cannot allocate device memory.
//
// diffattn_v2_decode needs a caller-provided workspace for its per-split partial results.
// Some callers cannot provide one: serving engines that hand nearly all HBM to a KV-cache
// pool or a caching allocator up front (a fresh cudaMalloc then fails, or forces the pool to
// give memory back), plugin interfaces that pass only input and output buffers, and loops
// that must not take the device-wide synchronisation cudaMalloc may imply. This entry point
// runs the same kernels with the partials in a fixed, statically sized device array that the
// library owns, so the call allocates nothing.
//
// The array is file-scope device memory: every GPU that loads this library holds it
// (kNoAllocScratchBytes) until the process exits. Host code cannot use the array's name as
// a device address (in host code it names a host-side stand-in), so its address is fetched
// with cudaGetSymbolAddress, once per device, with that device current, the first time the
// entry point runs on the device.

#include <mutex>

#include <cudaTypedefs.h>

#include "diffattn_v2.h"
#include "internal.h"

namespace {

// 16 MiB: enough for the partials of B*Hq*nsplit*(D+2) fp32 values of common decode batches
// (64 sequences x 64 heads at 8k context, or 8 sequences x 64 heads at 128k context).
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (set up once per device).
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    if (!p) return cudaErrorInvalidSymbol;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" int diffattn_v2_decode_noalloc(const void* q, const void* kcache, const void* vcache,
                                          const int32_t* seqlens, const float* lambda, void* out, int B,
                                          int Smax, int Hq, int Hkv, int D, da2_stream_t stream) {
  if (B < 0 || Smax <= 0 || D <= 0 || Hq <= 0 || Hkv <= 0 || (Hq % 2) != 0 || (Hq % (2 * Hkv)) != 0)
    return DA2_ERR_INVALID;
  if (B == 0) return DA2_OK;
  if (!q || !kcache || !vcache || !seqlens || !lambda || !out) return DA2_ERR_INVALID;
  if (!aligned16(q) || !aligned16(kcache) || !aligned16(vcache) || !aligned16(seqlens) || !aligned16(lambda) ||
      !aligned16(out))
    return DA2_ERR_INVALID;
  const int group = Hq / Hkv;
  if (D != 128 || !(group == 2 || group == 4 || group == 8 || group == 16)) return DA2_ERR_UNSUPPORTED;
  if (B > 65535 || Hkv > 65535) return DA2_ERR_UNSUPPORTED;
  // sizes whose partials do not fit the fixed array are refused, never truncated
  const size_t need = diffattn_v2_decode_workspace_size(B, Smax, Hq, Hkv, D);
  if (need == 0 || need > kNoAllocScratchBytes) return DA2_ERR_UNSUPPORTED;

  void* scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return DA2_ERR_CUDA;
  int* err = nullptr;
  if (da2::device_error_word(&err) != cudaSuccess) return DA2_ERR_CUDA;
  int split_len = 0, nsplit = 0;
  da2::decode_split_plan(B, Smax, Hkv, &split_len, &nsplit);
  CUtensorMap tk, tv;
  if (da2::encode_bshd_bf16(&tk, kcache, D, Hkv, Smax, B, 64, 64) != cudaSuccess) return DA2_ERR_CUDA;
  if (da2::encode_bshd_bf16(&tv, vcache, D, Hkv, Smax, B, 64, 64) != cudaSuccess) return DA2_ERR_CUDA;
  // The layout of diffattn_v2_decode's workspace, from the same helper. Nothing in it has to
  // start at zero: the split kernel writes every partial that the merge reads, and the
  // launch zeroes the split counters on the stream first.
  const da2::DecodeWorkspace ws = da2::decode_workspace_layout(scratch, B, 1, Hq, D, nsplit);
  cudaError_t e = da2::launch_decode(tk, tv, static_cast<const __nv_bfloat16*>(q), seqlens, lambda,
                                     static_cast<__nv_bfloat16*>(out), ws.o, ws.ml, ws.counters, err, B, Smax, Hq, Hkv,
                                     nsplit,
                                     split_len, nullptr, 0, 0, 1, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? DA2_OK : DA2_ERR_CUDA;
}
