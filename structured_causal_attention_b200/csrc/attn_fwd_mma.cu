// attn_fwd_mma.cu - Stream-Factorized attention forward, warp-level mma.sync path.
//
// Computes, for every query row r of a problem (see AttnParams in hd_common.cuh),
//   O_r = sum_c softmax_c(scale * q_r . k_c) v_c  over visible keys c, and LSE_r.
// Source: page "微信WeLM提出Hidden Decoding：大模型推理新范式" (tahou.com), section
// "规模化落地的工程优化" (intra-stream / cross-stream layers, KV-mirror) and
// section "隐式序列缩放的技术细节" step 2 (causal attention over the expanded
// sequence).
//
// Design: one CTA per (query tile of 128 rows, batch, head, stream group), 8
// warps x 16 rows. K/V tiles of 64 keys stream through a two-stage cp.async ring
// in XOR-swizzled shared memory; S = Q K^T and O += P V use m16n8k16 bf16 MMAs
// with fp32 accumulation; online softmax in base 2 with quad shuffles. Only the
// key tiles some row of the query tile can see are visited, and the mask is
// evaluated only on tiles that straddle the visibility boundary. INTRA problems
// are de-interleaved by address arithmetic (row stride n), so each stream is a
// contiguous causal problem.
#include "hd_common.cuh"
#include "launch.h"

namespace hd {

namespace {

constexpr int kFwdBM = 128;
constexpr int kFwdBN = 64;
constexpr int kFwdWarps = 8;
constexpr int kFwdThreads = kFwdWarps * 32;

template <int D>
struct FwdSmem {
  static constexpr int RC = D / 8;                      // 16-byte chunks per row
  static constexpr int Q_BYTES = kFwdBM * D * 2;
  static constexpr int KV_BYTES = kFwdBN * D * 2;
  static constexpr int TOTAL = Q_BYTES + 4 * KV_BYTES;  // Q + 2 x (K, V)
};

template <int D>
__global__ void __launch_bounds__(kFwdThreads, 1) attn_fwd_mma_kernel(const AttnParams p) {
  using SM = FwdSmem<D>;
  constexpr int RC = SM::RC;
  constexpr int NKT = kFwdBN / 8;  // n-tiles of S per warp
  constexpr int NDT = D / 8;       // n-tiles of O per warp
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* sQ = smem;
  uint8_t* sK = smem + SM::Q_BYTES;
  uint8_t* sV = sK + 2 * SM::KV_BYTES;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bhg = p.B * p.Hq * p.groups;
  const int num_qt = (p.Lq + kFwdBM - 1) / kFwdBM;
  const int qt = num_qt - 1 - static_cast<int>(blockIdx.x / bhg);  // heavy tiles first
  int y = static_cast<int>(blockIdx.x % bhg);
  const int grp = y % p.groups;
  y /= p.groups;
  const int h = y % p.Hq;
  const int b = y / p.Hq;
  const int hk = h / (p.Hq / p.Hkv);

  const int r0 = qt * kFwdBM;
  const int r_last = min(r0 + kFwdBM, p.Lq) - 1;
  const long long q_row0 = static_cast<long long>(b) * p.Sq + static_cast<long long>(grp) * p.qs_step;
  const long long k_row0 =
      static_cast<long long>(b) * p.S + static_cast<long long>(grp) * p.ks_step + p.ks_base;
  const __nv_bfloat16* qg = p.q + (q_row0 * p.Hq + h) * D;
  __nv_bfloat16* og = p.o + (q_row0 * p.Hq + h) * D;
  const long long q_rs = static_cast<long long>(p.q_rstride) * p.Hq * D;
  const __nv_bfloat16* kg = p.k + (k_row0 * p.Hkv + hk) * D;
  const __nv_bfloat16* vg = p.v + (k_row0 * p.Hkv + hk) * D;
  const long long k_rs = static_cast<long long>(p.k_rstride) * p.Hkv * D;

  // keys some row of this tile can see
  const int kmax = min(p.Lk - 1, p.a * r_last + p.bb);
  const int kmin = max(0, p.a * r0 + p.bb - p.win + 1);
  const int kt_lo = kmin / kFwdBN, kt_hi = kmax / kFwdBN;

  // ---- Q tile
  for (int i = tid; i < kFwdBM * RC; i += kFwdThreads) {
    const int row = i / RC, ch = i % RC, r = r0 + row;
    const __nv_bfloat16* src = qg + static_cast<long long>(min(r, p.Lq - 1)) * q_rs + ch * 8;
    cp_async16(smem_u32(sQ) + swz(row, ch, RC), src, r < p.Lq ? 16 : 0);
  }
  auto load_kv = [&](int kt, int st) {
    const int c0 = kt * kFwdBN;
    const uint32_t dk = smem_u32(sK + st * SM::KV_BYTES), dv = smem_u32(sV + st * SM::KV_BYTES);
    for (int i = tid; i < kFwdBN * RC; i += kFwdThreads) {
      const int row = i / RC, ch = i % RC, c = c0 + row;
      const long long off = static_cast<long long>(min(c, p.Lk - 1)) * k_rs + ch * 8;
      const int nb = c < p.Lk ? 16 : 0;
      cp_async16(dk + swz(row, ch, RC), kg + off, nb);
      cp_async16(dv + swz(row, ch, RC), vg + off, nb);
    }
  };
  load_kv(kt_lo, 0);
  cp_async_commit();

  uint32_t qf[D / 16][4];
  float o[NDT][4];
#pragma unroll
  for (int j = 0; j < NDT; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
  float m_run[2] = {-INFINITY, -INFINITY};
  float l_run[2] = {0.f, 0.f};
  const int wrow = warp * 16;

  for (int kt = kt_lo; kt <= kt_hi; ++kt) {
    const int st = (kt - kt_lo) & 1;
    if (kt < kt_hi) load_kv(kt + 1, st ^ 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    if (kt == kt_lo) {
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk)
        ldsm_x4(smem_u32(sQ) + swz(wrow + (lane & 15), kk * 2 + (lane >> 4), RC), qf[kk][0],
                qf[kk][1], qf[kk][2], qf[kk][3]);
    }
    const uint32_t kbase = smem_u32(sK + st * SM::KV_BYTES);
    const uint32_t vbase = smem_u32(sV + st * SM::KV_BYTES);

    // ---- S = Q K^T  (16 rows x 64 keys per warp)
    float s[NKT][4];
#pragma unroll
    for (int j = 0; j < NKT; ++j) s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
      for (int jp = 0; jp < NKT / 2; ++jp) {
        uint32_t b0, b1, b2, b3;
        const int key = jp * 16 + (lane & 7) + ((lane >> 4) << 3);
        ldsm_x4(kbase + swz(key, kk * 2 + ((lane >> 3) & 1), RC), b0, b1, b2, b3);
        mma_bf16_16816(s[2 * jp], qf[kk], b0, b1);
        mma_bf16_16816(s[2 * jp + 1], qf[kk], b2, b3);
      }
    }

    // ---- mask on boundary tiles only
    const int c0 = kt * kFwdBN;
    const bool full = (c0 + kFwdBN - 1 <= p.a * r0 + p.bb) &&
                      (c0 > p.a * r_last + p.bb - p.win) && (c0 + kFwdBN <= p.Lk);
    if (!full) {
#pragma unroll
      for (int j = 0; j < NKT; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int r = r0 + wrow + (lane >> 2) + ((e >> 1) << 3);
          const int c = c0 + j * 8 + (lane & 3) * 2 + (e & 1);
          if (!key_visible(p, r, c)) s[j][e] = -INFINITY;
        }
    }

    // ---- online softmax (base 2), rows lane/4 and lane/4 + 8
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      float mx = -INFINITY;
#pragma unroll
      for (int j = 0; j < NKT; ++j) mx = fmaxf(mx, fmaxf(s[j][2 * hr], s[j][2 * hr + 1]));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const float m_new = fmaxf(m_run[hr], mx * p.scale_log2);
      const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
      const float alpha = fast_exp2(m_run[hr] - m_use);
      m_run[hr] = m_new;
      float rs = 0.f;
#pragma unroll
      for (int j = 0; j < NKT; ++j) {
        const float p0 = fast_exp2(fmaf(s[j][2 * hr], p.scale_log2, -m_use));
        const float p1 = fast_exp2(fmaf(s[j][2 * hr + 1], p.scale_log2, -m_use));
        s[j][2 * hr] = p0;
        s[j][2 * hr + 1] = p1;
        rs += p0 + p1;
      }
      l_run[hr] = l_run[hr] * alpha + rs;
#pragma unroll
      for (int j = 0; j < NDT; ++j) {
        o[j][2 * hr] *= alpha;
        o[j][2 * hr + 1] *= alpha;
      }
    }

    // ---- O += P V
#pragma unroll
    for (int kk = 0; kk < kFwdBN / 16; ++kk) {
      uint32_t a[4];
      a[0] = pack_bf16(s[2 * kk][0], s[2 * kk][1]);
      a[1] = pack_bf16(s[2 * kk][2], s[2 * kk][3]);
      a[2] = pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
      a[3] = pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
      for (int dp = 0; dp < D / 16; ++dp) {
        uint32_t b0, b1, b2, b3;
        const int key = kk * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
        ldsm_x4_t(vbase + swz(key, dp * 2 + (lane >> 4), RC), b0, b1, b2, b3);
        mma_bf16_16816(o[2 * dp], a, b0, b1);
        mma_bf16_16816(o[2 * dp + 1], a, b2, b3);
      }
    }
    __syncthreads();
  }
  cp_async_wait<0>();

  // ---- epilogue: normalise, LSE, O through shared memory (own rows only)
#pragma unroll
  for (int hr = 0; hr < 2; ++hr) {
    float l = l_run[hr];
    l += __shfl_xor_sync(0xffffffffu, l, 1);
    l += __shfl_xor_sync(0xffffffffu, l, 2);
    const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
    for (int j = 0; j < NDT; ++j) {
      o[j][2 * hr] *= inv;
      o[j][2 * hr + 1] *= inv;
    }
    const int row = wrow + (lane >> 2) + hr * 8;
    const int r = r0 + row;
    if ((lane & 3) == 0 && r < p.Lq) {
      const long long li = (static_cast<long long>(b) * p.Hq + h) * p.Sq +
                           static_cast<long long>(grp) * p.qs_step +
                           static_cast<long long>(r) * p.q_rstride;
      p.lse[li] = (m_run[hr] + __log2f(l)) * 0.69314718055994530942f;
    }
#pragma unroll
    for (int j = 0; j < NDT; ++j) {
      const int col = j * 8 + (lane & 3) * 2;
      *reinterpret_cast<uint32_t*>(sQ + swz(row, col >> 3, RC) + (col & 7) * 2) =
          pack_bf16(o[j][2 * hr], o[j][2 * hr + 1]);
    }
  }
  __syncwarp();
  for (int i = lane; i < 16 * RC; i += 32) {
    const int row = i / RC, ch = i % RC, r = r0 + wrow + row;
    if (r < p.Lq)
      *reinterpret_cast<uint4*>(og + static_cast<long long>(r) * q_rs + ch * 8) =
          *reinterpret_cast<const uint4*>(sQ + swz(wrow + row, ch, RC));
  }
}

template <int D>
cudaError_t launch_fwd_d(const AttnParams& p, cudaStream_t stream) {
  const int smem = FwdSmem<D>::TOTAL;
  cudaError_t e = cudaFuncSetAttribute(attn_fwd_mma_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const long long num_qt = (p.Lq + kFwdBM - 1) / kFwdBM;
  const long long blocks = num_qt * p.B * p.Hq * p.groups;
  attn_fwd_mma_kernel<D><<<static_cast<unsigned>(blocks), kFwdThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_fwd_mma(const AttnParams& p, cudaStream_t stream) {
  if (p.D == 64) return launch_fwd_d<64>(p, stream);
  if (p.D == 128) return launch_fwd_d<128>(p, stream);
  return cudaErrorInvalidValue;
}

}  // namespace hd
