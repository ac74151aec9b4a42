// expand.cu - interleaved n-table embedding gather.
//
// Page "微信WeLM提出Hidden Decoding：大模型推理新范式" (tahou.com), section
// "隐式序列缩放的技术细节", step 1: with n embedding tables, stream k of token i
// is placed at physical position (i-1)n+k of the nL-long expanded sequence.
// 0-based: out[b, t*n + s, :] = tables[s, ids[b, t], :].
//
// A pure byte copy (HBM-bound): one warp per output row, 16-byte vector loads
// and stores when the row length allows, all of a lane's loads issued before
// its stores. A token id outside [0, V) leaves the row zero and records
// HD_ERR_DEVICE_INDEX.
#include "hd_common.cuh"
#include "launch.h"

namespace hd {

namespace {

template <typename Vec, int UNROLL>
__global__ void __launch_bounds__(256) expand_kernel(const int32_t* __restrict__ ids,
                                                     const uint8_t* __restrict__ tables,
                                                     uint8_t* __restrict__ out, int B, int L,
                                                     int n, int V, long long row_bytes,
                                                     int* status) {
  const long long nrows = static_cast<long long>(B) * L * n;
  const int lane = threadIdx.x & 31;
  const long long warps = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
  const long long nvec = row_bytes / static_cast<long long>(sizeof(Vec));
  for (long long row = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
       row < nrows; row += warps) {
    const int s = static_cast<int>(row % n);
    const long long bt = row / n;  // b*L + t
    const int id = __ldg(ids + bt);
    Vec* dst = reinterpret_cast<Vec*>(out + row * row_bytes);
    if (id < 0 || id >= V) {
      if (lane == 0) record_status(status, HD_ERR_DEVICE_INDEX);
      Vec z;
      memset(&z, 0, sizeof(Vec));
      for (long long i = lane; i < nvec; i += 32) dst[i] = z;
      continue;
    }
    if (!in_bounds((static_cast<long long>(s) * V + id) * row_bytes, row_bytes,
                   static_cast<long long>(n) * V * row_bytes, status) ||
        !in_bounds(row * row_bytes, row_bytes, nrows * row_bytes, status))
      continue;
    const Vec* src = reinterpret_cast<const Vec*>(
        tables + (static_cast<long long>(s) * V + id) * row_bytes);
    long long i = lane;
    for (; i + 32 * (UNROLL - 1) < nvec; i += 32 * UNROLL) {
      Vec r[UNROLL];
#pragma unroll
      for (int u = 0; u < UNROLL; ++u) r[u] = __ldg(src + i + 32 * u);
#pragma unroll
      for (int u = 0; u < UNROLL; ++u) dst[i + 32 * u] = r[u];
    }
    for (; i < nvec; i += 32) dst[i] = __ldg(src + i);
  }
}

template <typename Vec, int UNROLL>
cudaError_t launch_vec(const int32_t* ids, const void* tables, void* out, int B, int L, int n,
                       int V, long long row_bytes, int sms, int* status, cudaStream_t stream) {
  const long long nrows = static_cast<long long>(B) * L * n;
  long long blocks = (nrows + 7) / 8;
  const long long cap = static_cast<long long>(sms) * 8 * 16;  // grid-stride beyond 16 waves of 8 warps
  if (blocks > cap) blocks = cap;
  expand_kernel<Vec, UNROLL><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
      ids, static_cast<const uint8_t*>(tables), static_cast<uint8_t*>(out), B, L, n, V, row_bytes,
      status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_expand(const int32_t* ids, const void* tables, void* out, int B, int L, int n,
                          int V, long long row_bytes, int sms, int* status, cudaStream_t stream) {
  const bool a16 = (reinterpret_cast<uintptr_t>(tables) % 16 == 0) &&
                   (reinterpret_cast<uintptr_t>(out) % 16 == 0) && (row_bytes % 16 == 0);
  if (a16) return launch_vec<uint4, 4>(ids, tables, out, B, L, n, V, row_bytes, sms, status, stream);
  const bool a4 = (reinterpret_cast<uintptr_t>(tables) % 4 == 0) &&
                  (reinterpret_cast<uintptr_t>(out) % 4 == 0) && (row_bytes % 4 == 0);
  if (a4) return launch_vec<uint32_t, 4>(ids, tables, out, B, L, n, V, row_bytes, sms, status, stream);
  return launch_vec<uint16_t, 4>(ids, tables, out, B, L, n, V, row_bytes, sms, status, stream);
}

}  // namespace hd
