// attn_bwd.cu - Stream-Factorized attention backward: launch sequence and the
// small element-wise kernels around the tensor-core main kernel.
//
// Gradients of O = softmax(scale Q K^T over visible keys) V (page "微信WeLM提出
// Hidden Decoding：大模型推理新范式", tahou.com, section "规模化落地的工程优化"):
//   D_i = sum_d dO_id O_id,  P_ij = exp(scale q_i.k_j - LSE_i),
//   dP = dO V^T,  dS = P * (dP - D),
//   dQ = scale dS K,  dK = scale sum_group dS^T Q,  dV = sum_group P^T dO.
//
// Kernels on the caller's stream:
//   1. bwd_pre:   D = rowsum(dO * O) and LSE * log2(e), both packed per
//                 problem (row-contiguous, padded to 64 rows); zero the fp32 dQ
//                 accumulator.
//   2. attn_bwd_tc_kernel (attn_bwd_tc.cu): dK, dV and the fp32 dQ sums.
//   3. bwd_zero_unread_kv (INTRA with final-stream-only queries only): the dK /
//                 dV rows of streams 0..n-2, which no query reads, are zero.
//   4. bwd_dq:    dQ = bf16(scale * accumulator).
#include "hd_common.cuh"
#include "launch.h"

namespace hd {

namespace {

// D = rowsum(dO * O) and LSE * log2(e), packed per problem; the fp32 dQ
// accumulator zeroed. D/8 lanes per row (16-byte loads of 8 bf16 each), so a
// warp covers 32 / (D/8) rows per pass.
template <int D>
__global__ void __launch_bounds__(256) bwd_pre_kernel(const AttnParams p) {
  constexpr int LPR = D / 8;           // lanes per row
  constexpr int RPW = 32 / LPR;        // rows per warp
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sub = lane / LPR, sl = lane % LPR;
  const long long row = (static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + warp) * RPW + sub;
  const long long total = static_cast<long long>(p.B) * p.Sq * p.Hq;
  const bool valid = row < total && in_bounds(row * D + 8 * sl, 8, p.ext_q, p.status);
  float acc = 0.f;
  if (valid) {
    const uint4 ov = __ldcs(reinterpret_cast<const uint4*>(p.o + row * D) + sl);
    const uint4 gv = __ldcs(reinterpret_cast<const uint4*>(p.dout + row * D) + sl);
    const uint32_t* o2 = reinterpret_cast<const uint32_t*>(&ov);
    const uint32_t* g2 = reinterpret_cast<const uint32_t*>(&gv);
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const float2 of = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&o2[w]));
      const float2 gf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&g2[w]));
      acc = fmaf(of.x, gf.x, acc);
      acc = fmaf(of.y, gf.y, acc);
    }
  }
#pragma unroll
  for (int s = LPR / 2; s > 0; s >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, s);
  if (!valid) return;
  const int h = static_cast<int>(row % p.Hq);
  const long long bi = row / p.Hq;
  const long long i = bi % p.Sq, b = bi / p.Sq;
  // packed row statistics of problem (b, h, grp), row r
  const bool intra_groups = p.mode == HD_INTRA && !p.final_only;
  const long long grp = intra_groups ? i % p.n : 0;
  const long long r = intra_groups ? i / p.n : i;
  const long long pk = ((b * p.Hq + h) * p.groups + grp) * p.lq_pad;
  if (sl == 0 && in_bounds(pk + r, 1, p.ext_packed, p.status) &&
      in_bounds((b * p.Hq + h) * p.Sq + i, 1, p.ext_lse, p.status)) {
    p.deltap[pk + r] = acc;
    p.lse2p[pk + r] = p.lse[(b * p.Hq + h) * p.Sq + i] * 1.4426950408889634074f;
  }
  if (r == p.Lq - 1) {  // zero the padding rows after the problem's last row
    for (int j = sl; j < p.lq_pad - p.Lq; j += LPR) {
      if (!in_bounds(pk + p.Lq + j, 1, p.ext_packed, p.status)) break;
      p.deltap[pk + p.Lq + j] = 0.f;
      p.lse2p[pk + p.Lq + j] = 0.f;
    }
  }
  float4* z = reinterpret_cast<float4*>(p.dq_acc + row * D) + 2 * sl;
  z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
  z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// INTRA with final-stream-only queries: only stream n-1's keys are read, so
// the dK / dV rows of streams 0..n-2 are exactly zero.
__global__ void bwd_zero_unread_kv_kernel(const AttnParams p) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long row = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + warp;  // (b, pos, hk)
  const long long total = static_cast<long long>(p.B) * p.S * p.Hkv;
  if (row >= total) return;
  const long long pos = (row / p.Hkv) % p.S;
  if (pos % p.n == p.n - 1) return;
  if (!in_bounds(row * p.D, p.D, p.ext_kv, p.status)) return;
  uint2* zk = reinterpret_cast<uint2*>(p.dk + row * p.D);
  uint2* zv = reinterpret_cast<uint2*>(p.dv + row * p.D);
  for (int c = lane; c < p.D / 4; c += 32) {
    zk[c] = make_uint2(0u, 0u);
    zv[c] = make_uint2(0u, 0u);
  }
}

__global__ void bwd_dq_kernel(const AttnParams p, long long n8) {
  const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n8 || !in_bounds(8 * i, 8, p.ext_q, p.status)) return;
  const float4 a = reinterpret_cast<const float4*>(p.dq_acc)[2 * i];
  const float4 c = reinterpret_cast<const float4*>(p.dq_acc)[2 * i + 1];
  uint4 out;
  out.x = pack_bf16(a.x * p.scale, a.y * p.scale);
  out.y = pack_bf16(a.z * p.scale, a.w * p.scale);
  out.z = pack_bf16(c.x * p.scale, c.y * p.scale);
  out.w = pack_bf16(c.z * p.scale, c.w * p.scale);
  reinterpret_cast<uint4*>(p.dq)[i] = out;
}

}  // namespace

cudaError_t launch_attn_bwd(const AttnParams& p, cudaStream_t stream) {
  if (p.D != 64 && p.D != 128) return cudaErrorInvalidValue;
  const long long rows = static_cast<long long>(p.B) * p.Sq * p.Hq;
  const long long rows_per_block = 8 * (32 / (p.D / 8));  // 8 warps
  const unsigned pre_blocks = static_cast<unsigned>((rows + rows_per_block - 1) / rows_per_block);
  if (p.D == 64) bwd_pre_kernel<64><<<pre_blocks, 256, 0, stream>>>(p);
  else bwd_pre_kernel<128><<<pre_blocks, 256, 0, stream>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = launch_attn_bwd_tc_main(p, stream);
  if (e != cudaSuccess) return e;
  if (p.mode == HD_INTRA && p.final_only && p.n > 1) {
    const long long kv_rows = static_cast<long long>(p.B) * p.S * p.Hkv;
    bwd_zero_unread_kv_kernel<<<static_cast<unsigned>((kv_rows + 7) / 8), 256, 0, stream>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  const long long n8 = rows * p.D / 8;
  bwd_dq_kernel<<<static_cast<unsigned>((n8 + 255) / 256), 256, 0, stream>>>(p, n8);
  return cudaGetLastError();
}

}  // namespace hd
