// decode_noalloc.cu - hd_decode_attn_noalloc: the decode step of hd_decode_attn
// with its split-K scratch held by the library itself instead of passed in.
//
// Who needs it: code that may not allocate device memory when it runs a decode
// step - for example a serving loop whose host framework owns every byte of the
// GPU through its own pool and forbids other allocations, or a latency-bound
// loop that must never enter cudaMalloc, which can block on or synchronise the
// device. Such a caller still owns the inputs and outputs; only the scratch
// moves into a fixed array compiled into this library.
//
// The scratch is one file-scope __device__ array of HD_DECODE_NOALLOC_SCRATCH_BYTES.
// Every GPU that loads the library holds it until the process exits. All calls
// on a device share it and it keeps whatever the last call left there; the
// decode kernels write every partial they later read within the same call, so
// nothing needs clearing between calls. Two calls that run at the same time on
// one device (two streams, or two host threads without ordering) race on the
// array and corrupt each other's results: order such calls on one stream or
// with events.
#include "hd_common.cuh"
#include "launch.h"

namespace hd {
namespace {

static __device__ __align__(256) unsigned char g_decode_scratch[HD_DECODE_NOALLOC_SCRATCH_BYTES];

// Device address of the scratch on the current device. In host code the
// symbol names a host-side stand-in, not device memory, so the address is
// looked up with the calling device current. The lookup is repeated on every
// call (a map lookup in the runtime), so it never goes stale, not even after
// a device reset.
int scratch_address(void** out) {
  void* ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_decode_scratch) != cudaSuccess || !ptr) return HD_ERR_CUDA;
  *out = ptr;
  return HD_OK;
}

}  // namespace
}  // namespace hd

extern "C" int hd_decode_attn_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                      const int32_t* seqlen, void* out, float* lse, int B, int n,
                                      int Tcap, int Hq, int Hkv, int D, int mode, int W_tokens,
                                      float scale, void* stream) {
  const size_t need = hd_decode_workspace_bytes(B, n, Tcap, Hq, Hkv, D);
  if (need == 0) return HD_ERR_INVALID_ARG;
  if (need > static_cast<size_t>(HD_DECODE_NOALLOC_SCRATCH_BYTES)) return HD_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  const int st = hd::scratch_address(&scratch);
  if (st != HD_OK) return st;
  return hd_decode_attn(q, k_cache, v_cache, seqlen, out, lse, B, n, Tcap, Hq, Hkv, D, mode,
                        W_tokens, scale, scratch, static_cast<size_t>(HD_DECODE_NOALLOC_SCRATCH_BYTES),
                        stream);
}
