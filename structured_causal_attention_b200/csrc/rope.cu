// rope.cu - rotary position embedding at the physical expanded positions.
//
// Page "微信WeLM提出Hidden Decoding：大模型推理新范式" (tahou.com), section
// "隐式序列缩放的技术细节", step 2: the expanded sequence keeps the base model's
// position encoding, continued over all n*L positions, so stream s of token t
// is encoded at p = (t0 + t)*n + s, t0 being the tokens that precede the call
// (0 for a prefill, the cache length for a decode step). Rotate-half pairing:
//   x[i]     <- x[i] cos(p w_i) - x[i+D/2] sin(p w_i)
//   x[i+D/2] <- x[i+D/2] cos(p w_i) + x[i] sin(p w_i),   w_i = base^(-2i/D).
//
// In place and HBM-bound (one read and one write of every element). A thread
// owns one block of 8 frequencies of one row and walks all heads of that row,
// so each sin/cos pair is computed once per row and reused H times. The grid
// stride is a multiple of D/16, so a thread's frequency block never changes
// and its w_i are computed once. Angles are formed and reduced to [-pi, pi] in
// float64 (p*w_i reaches 1e5 rad and more), then evaluated with the float32
// hardware approximation, whose absolute error on [-pi, pi] is below 4e-7.
#include "hd_common.cuh"
#include "launch.h"

namespace hd {

namespace {

constexpr int kRopeThreads = 256;
constexpr int kRopeUnroll = 4;  // heads whose loads are in flight together

__device__ __forceinline__ void rotate8(uint4& lo, uint4& hi, const float* c, const float* s) {
  uint32_t* a = reinterpret_cast<uint32_t*>(&lo);
  uint32_t* b = reinterpret_cast<uint32_t*>(&hi);
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    const float2 x1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&a[w]));
    const float2 x2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&b[w]));
    const float c0 = c[2 * w], c1 = c[2 * w + 1], s0 = s[2 * w], s1 = s[2 * w + 1];
    const __nv_bfloat162 o1 =
        __floats2bfloat162_rn(fmaf(x1.x, c0, -x2.x * s0), fmaf(x1.y, c1, -x2.y * s1));
    const __nv_bfloat162 o2 =
        __floats2bfloat162_rn(fmaf(x2.x, c0, x1.x * s0), fmaf(x2.y, c1, x1.y * s1));
    a[w] = *reinterpret_cast<const uint32_t*>(&o1);
    b[w] = *reinterpret_cast<const uint32_t*>(&o2);
  }
}

// Rotates the H heads of one row (row base `x`, head stride D elements).
__device__ __forceinline__ void rotate_row(__nv_bfloat16* x, int H, int D, int j, const float* c,
                                           const float* s) {
  const int half = D / 2;
  uint4* base_lo = reinterpret_cast<uint4*>(x + j * 8);
  uint4* base_hi = reinterpret_cast<uint4*>(x + half + j * 8);
  const int hstride = D / 8;  // uint4 per head
  int h = 0;
  for (; h + kRopeUnroll <= H; h += kRopeUnroll) {
    uint4 lo[kRopeUnroll], hi[kRopeUnroll];
#pragma unroll
    for (int u = 0; u < kRopeUnroll; ++u) {
      lo[u] = __ldcs(base_lo + (h + u) * hstride);
      hi[u] = __ldcs(base_hi + (h + u) * hstride);
    }
#pragma unroll
    for (int u = 0; u < kRopeUnroll; ++u) {
      rotate8(lo[u], hi[u], c, s);
      __stcs(base_lo + (h + u) * hstride, lo[u]);
      __stcs(base_hi + (h + u) * hstride, hi[u]);
    }
  }
  for (; h < H; ++h) {
    uint4 lo = __ldcs(base_lo + h * hstride), hi = __ldcs(base_hi + h * hstride);
    rotate8(lo, hi, c, s);
    __stcs(base_lo + h * hstride, lo);
    __stcs(base_hi + h * hstride, hi);
  }
}

// Tasks [0, nq) rotate query rows, [nq, nq + nk) key rows; task = row*J + j.
__global__ void __launch_bounds__(kRopeThreads) rope_kernel(RopeParams p) {
  const int J = p.D / 16;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;  // multiple of J
  long long task = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int j = static_cast<int>(task % J);
  double w[8];
#pragma unroll
  for (int e = 0; e < 8; ++e)
    w[e] = exp2(-static_cast<double>(2 * (j * 8 + e)) / p.D * p.log2_base);
  const long long nq = p.q ? static_cast<long long>(p.B) * p.Sq * J : 0;
  const long long nk = p.k ? static_cast<long long>(p.B) * p.S * J : 0;
  const double kTwoPi = 6.283185307179586;
  const double kInvTwoPi = 0.15915494309189535;
  for (; task < nq + nk; task += stride) {
    const bool is_q = task < nq;
    const long long row = (is_q ? task : task - nq) / J;  // b*rows + r
    const int rows = is_q ? p.Sq : p.S;
    const int b = static_cast<int>(row / rows);
    const int r = static_cast<int>(row % rows);
    const long long t0 = p.token_offset ? static_cast<long long>(p.token_offset[b]) : 0;
    if (t0 < 0) {
      if (j == 0) record_status(p.status, HD_ERR_DEVICE_INDEX);
      continue;
    }
    // Physical position of the row: q rows of a final-stream-only call are the
    // streams n-1 of consecutive tokens; all other rows are consecutive positions.
    const long long pos = (is_q && p.final_only) ? (t0 + r) * p.n + (p.n - 1) : t0 * p.n + r;
    float c[8], s[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const double a = static_cast<double>(pos) * w[e];
      const double red = fma(-rint(a * kInvTwoPi), kTwoPi, a);
      __sincosf(static_cast<float>(red), &s[e], &c[e]);  // abs error < 4e-7 on [-pi, pi]
    }
    const int H = is_q ? p.Hq : p.Hkv;
    const long long ext = static_cast<long long>(p.B) * rows * H * p.D;
    if (!in_bounds(row * H * p.D, static_cast<long long>(H) * p.D, ext, p.status)) continue;
    __nv_bfloat16* x = (is_q ? p.q : p.k) + row * H * p.D;
    rotate_row(x, H, p.D, j, c, s);
  }
}

}  // namespace

cudaError_t launch_rope(const RopeParams& p, int sms, cudaStream_t stream) {
  const int J = p.D / 16;
  const long long tasks = (p.q ? static_cast<long long>(p.B) * p.Sq * J : 0) +
                          (p.k ? static_cast<long long>(p.B) * p.S * J : 0);
  long long blocks = (tasks + kRopeThreads - 1) / kRopeThreads;
  const long long cap = static_cast<long long>(sms) * 8;  // 8 resident 256-thread blocks per SM, grid-stride beyond
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  static_assert(kRopeThreads % 16 == 0, "the grid stride must be a multiple of D/16 <= 16");
  rope_kernel<<<static_cast<unsigned>(blocks), kRopeThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace hd
