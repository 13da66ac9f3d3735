// ssa_decode_noalloc: the decode step with its scratch in a fixed device array
// of the library instead of a caller-supplied workspace, for callers that
// cannot allocate device memory when they call.  Same kernels and results as
// ssa_decode.
#include <mutex>

#include <cuda_runtime.h>

#include "kernels.h"
#include "ssa.h"

// One scratch area per device, held from module load until the process exits.
// Host code must not use this name as an address: it is a host-side shadow.
// The device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char ssa_decode_scratch[SSA_DECODE_NOALLOC_MAX_BYTES];

namespace {

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of ssa_decode_scratch on the current device, looked up once
// per device (with that device current) and cached.
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, ssa_decode_scratch);
    if (e != cudaSuccess) return e;
    if (p == nullptr) return cudaErrorInvalidSymbol;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" ssa_status ssa_decode_noalloc(const void* q, const void* Kc, const void* Vc,
                                         ssa_dtype dtype, const float* S,
                                         const int32_t* seqlens, int batch, int Hq, int Hkv,
                                         int Lmax, int d, int B, int topk, float scale, void* O,
                                         int32_t* idx, ssa_stream stream) {
  if (dtype != SSA_F32 && dtype != SSA_BF16) return SSA_ERR_INVALID_ARG;
  if (B <= 0 || d <= 0) return SSA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return SSA_ERR_UNSUPPORTED;
  if (B % 16 != 0 || B > 128) return SSA_ERR_UNSUPPORTED;
  if (batch <= 0 || Hq <= 0 || Hkv <= 0 || Lmax <= 0 || topk < 0) return SSA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return SSA_ERR_INVALID_ARG;
  if (Hq / Hkv > 8) return SSA_ERR_UNSUPPORTED;
  if (Lmax / B > 16384) return SSA_ERR_UNSUPPORTED;
  if (!(scale > 0.f)) return SSA_ERR_INVALID_ARG;
  if (q == nullptr || Kc == nullptr || Vc == nullptr || seqlens == nullptr || O == nullptr)
    return SSA_ERR_INVALID_ARG;
  if (Lmax / B > 0 && S == nullptr) return SSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(Kc) || !aligned16(Vc) || !aligned16(S) || !aligned16(O))
    return SSA_ERR_INVALID_ARG;
  const ssa::DecodePlan p = ssa::plan_decode(batch, Hq, Hkv, d, B, topk, Lmax);
  if (p.bytes > SSA_DECODE_NOALLOC_MAX_BYTES) return SSA_ERR_UNSUPPORTED;
  void* ws = nullptr;
  if (scratch_address(&ws) != cudaSuccess) return SSA_ERR_CUDA;
  // The split counters are zeroed by the routing launch of every call; every
  // other scratch word is written before it is read, so the previous call's
  // contents never leak into this one.
  const cudaError_t e =
      ssa::launch_decode(p, q, Kc, Vc, dtype, S, seqlens, batch, Hq, Hkv, Lmax, d, B, scale, O,
                         idx, ws, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SSA_OK : SSA_ERR_CUDA;
}
