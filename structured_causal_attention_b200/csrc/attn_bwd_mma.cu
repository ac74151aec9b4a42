// attn_bwd_mma.cu - Stream-Factorized attention backward, warp-level mma.sync path.
//
// Gradients of O = softmax(scale Q K^T over visible keys) V (page "微信WeLM提出
// Hidden Decoding：大模型推理新范式", tahou.com, section "规模化落地的工程优化"):
//   D_i = sum_d dO_id O_id,  P_ij = exp(scale q_i.k_j - LSE_i),
//   dP = dO V^T,  dS = P * (dP - D),
//   dQ = scale dS K,  dK = scale sum_group dS^T Q,  dV = sum_group P^T dO.
//
// Three kernels on the caller's stream:
//   1. bwd_pre:   D = rowsum(dO * O) (fp32, LSE layout); zero the fp32 dQ
//                 accumulator.
//   2. bwd_main:  one CTA per (64-key tile, batch, KV head, stream group). It
//                 loops over the query heads of the GQA group and the query
//                 tiles that can see its keys, recomputing S^T and P^T, and
//                 keeps dK / dV for its keys in registers (the group sum needs
//                 no atomics). dQ partials go to the fp32 accumulator with
//                 vector atomics.
//   3. bwd_dq:    dQ = bf16(scale * accumulator).
// With INTRA and final-stream-only queries a fourth kernel zeroes the dK / dV
// rows of streams 0..n-2, which no query reads.
#include "hd_common.cuh"
#include "launch.h"

namespace hd {

namespace {

constexpr int kBwdBN = 64;  // keys per CTA
constexpr int kBwdBM = 64;  // query rows per iteration
constexpr int kBwdWarps = 4;
constexpr int kBwdThreads = kBwdWarps * 32;
constexpr float kLog2e = 1.4426950408889634074f;

template <int D>
struct BwdSmem {
  static constexpr int RC = D / 8;
  static constexpr int TILE = 64 * D * 2;
  static constexpr int K_OFF = 0;
  static constexpr int V_OFF = TILE;
  static constexpr int Q_OFF = 2 * TILE;   // 2 stages
  static constexpr int DO_OFF = 4 * TILE;  // 2 stages
  static constexpr int DS_OFF = 6 * TILE;  // 64 x 64 bf16
  static constexpr int L_OFF = DS_OFF + 64 * 64 * 2;  // 2 x 64 fp32 (LSE, log2 units)
  static constexpr int DL_OFF = L_OFF + 2 * 64 * 4;   // 2 x 64 fp32 (D)
  static constexpr int TOTAL = DL_OFF + 2 * 64 * 4;
};

__global__ void bwd_pre_kernel(const AttnParams p) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long row = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + warp;
  const long long total = static_cast<long long>(p.B) * p.Sq * p.Hq;
  if (row >= total) return;
  const int h = static_cast<int>(row % p.Hq);
  const long long bi = row / p.Hq;
  const long long i = bi % p.Sq, b = bi / p.Sq;
  const __nv_bfloat16* o = p.o + row * p.D;
  const __nv_bfloat16* g = p.dout + row * p.D;
  float acc = 0.f;
  for (int c = lane * 2; c < p.D; c += 64) {
    const __nv_bfloat162 ov = *reinterpret_cast<const __nv_bfloat162*>(o + c);
    const __nv_bfloat162 gv = *reinterpret_cast<const __nv_bfloat162*>(g + c);
    acc = fmaf(__low2float(ov), __low2float(gv), acc);
    acc = fmaf(__high2float(ov), __high2float(gv), acc);
  }
#pragma unroll
  for (int s = 16; s > 0; s >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, s);
  if (lane == 0) p.delta[(b * p.Hq + h) * p.Sq + i] = acc;
  float4* z = reinterpret_cast<float4*>(p.dq_acc + row * p.D);
  for (int c = lane; c < p.D / 4; c += 32) z[c] = make_float4(0.f, 0.f, 0.f, 0.f);
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
  uint2* zk = reinterpret_cast<uint2*>(p.dk + row * p.D);
  uint2* zv = reinterpret_cast<uint2*>(p.dv + row * p.D);
  for (int c = lane; c < p.D / 4; c += 32) {
    zk[c] = make_uint2(0u, 0u);
    zv[c] = make_uint2(0u, 0u);
  }
}

__global__ void bwd_dq_kernel(const AttnParams p, long long n8) {
  const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n8) return;
  const float4 a = reinterpret_cast<const float4*>(p.dq_acc)[2 * i];
  const float4 c = reinterpret_cast<const float4*>(p.dq_acc)[2 * i + 1];
  uint4 out;
  out.x = pack_bf16(a.x * p.scale, a.y * p.scale);
  out.y = pack_bf16(a.z * p.scale, a.w * p.scale);
  out.z = pack_bf16(c.x * p.scale, c.y * p.scale);
  out.w = pack_bf16(c.z * p.scale, c.w * p.scale);
  reinterpret_cast<uint4*>(p.dq)[i] = out;
}

template <int D>
__global__ void __launch_bounds__(kBwdThreads, 2) bwd_main_kernel(const AttnParams p) {
  using SM = BwdSmem<D>;
  constexpr int RC = SM::RC;
  constexpr int NDT = D / 8;
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* sK = smem + SM::K_OFF;
  uint8_t* sV = smem + SM::V_OFF;
  float* sL = reinterpret_cast<float*>(smem + SM::L_OFF);
  float* sDl = reinterpret_cast<float*>(smem + SM::DL_OFF);
  const uint32_t sQ0 = smem_u32(smem + SM::Q_OFF);
  const uint32_t sO0 = smem_u32(smem + SM::DO_OFF);
  const uint32_t sS = smem_u32(smem + SM::DS_OFF);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bkg = p.B * p.Hkv * p.groups;
  const int kt = static_cast<int>(blockIdx.x / bkg);  // low key tiles see the most queries
  int y = static_cast<int>(blockIdx.x % bkg);
  const int grp = y % p.groups;
  y /= p.groups;
  const int hk = y % p.Hkv;
  const int b = y / p.Hkv;
  const int g = p.Hq / p.Hkv;

  const int c0 = kt * kBwdBN;
  const int c_last = min(c0 + kBwdBN, p.Lk) - 1;
  const long long q_row0 = static_cast<long long>(b) * p.Sq + static_cast<long long>(grp) * p.qs_step;
  const long long k_row0 =
      static_cast<long long>(b) * p.S + static_cast<long long>(grp) * p.ks_step + p.ks_base;
  const long long q_rs = static_cast<long long>(p.q_rstride) * p.Hq * D;
  const long long k_rs = static_cast<long long>(p.k_rstride) * p.Hkv * D;
  const __nv_bfloat16* kg = p.k + (k_row0 * p.Hkv + hk) * D;
  const __nv_bfloat16* vg = p.v + (k_row0 * p.Hkv + hk) * D;

  // query rows that can see some key of this tile
  const int rmin = (c0 - p.bb <= 0) ? 0 : (c0 - p.bb + p.a - 1) / p.a;
  const int rmax = min(p.Lq - 1, (c_last + p.win - 1 - p.bb) / p.a);
  const int qt_lo = rmin / kBwdBM, qt_hi = rmax / kBwdBM;
  const int nqt = rmin <= rmax ? qt_hi - qt_lo + 1 : 0;
  const int total_it = g * nqt;

  // K, V tiles
  for (int i = tid; i < kBwdBN * RC; i += kBwdThreads) {
    const int row = i / RC, ch = i % RC, c = c0 + row;
    const long long off = static_cast<long long>(min(c, p.Lk - 1)) * k_rs + ch * 8;
    cp_async16(smem_u32(sK) + swz(row, ch, RC), kg + off, c < p.Lk ? 16 : 0);
    cp_async16(smem_u32(sV) + swz(row, ch, RC), vg + off, c < p.Lk ? 16 : 0);
  }
  auto load_q = [&](int it, int st) {
    const int gi = it / nqt, qt = qt_lo + it % nqt, h = hk * g + gi;
    const __nv_bfloat16* qg = p.q + (q_row0 * p.Hq + h) * D;
    const __nv_bfloat16* dg = p.dout + (q_row0 * p.Hq + h) * D;
    const uint32_t dq = sQ0 + st * SM::TILE, dd = sO0 + st * SM::TILE;
    for (int i = tid; i < kBwdBM * RC; i += kBwdThreads) {
      const int row = i / RC, ch = i % RC, r = qt * kBwdBM + row;
      const long long off = static_cast<long long>(min(r, p.Lq - 1)) * q_rs + ch * 8;
      cp_async16(dq + swz(row, ch, RC), qg + off, r < p.Lq ? 16 : 0);
      cp_async16(dd + swz(row, ch, RC), dg + off, r < p.Lq ? 16 : 0);
    }
    if (tid < kBwdBM) {
      const int r = qt * kBwdBM + tid;
      float l2 = 0.f, dl = 0.f;
      if (r < p.Lq) {
        const long long li = (static_cast<long long>(b) * p.Hq + h) * p.Sq +
                             static_cast<long long>(grp) * p.qs_step +
                             static_cast<long long>(r) * p.q_rstride;
        l2 = p.lse[li] * kLog2e;
        dl = p.delta[li];
      }
      sL[st * 64 + tid] = l2;
      sDl[st * 64 + tid] = dl;
    }
  };
  if (total_it > 0) load_q(0, 0);
  cp_async_commit();

  float dk[NDT][4], dv[NDT][4];
#pragma unroll
  for (int j = 0; j < NDT; ++j)
#pragma unroll
    for (int e = 0; e < 4; ++e) dk[j][e] = dv[j][e] = 0.f;
  const int wk = warp * 16;  // this warp's keys within the tile

  for (int it = 0; it < total_it; ++it) {
    const int st = it & 1;
    if (it + 1 < total_it) load_q(it + 1, st ^ 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const int gi = it / nqt, qt = qt_lo + it % nqt, h = hk * g + gi;
    const int rq0 = qt * kBwdBM;
    const uint32_t sQ = sQ0 + st * SM::TILE, sO = sO0 + st * SM::TILE;

    // ---- S^T = K Q^T and dP^T = V dO^T (16 keys x 64 queries per warp)
    float sT[8][4], dpT[8][4];
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) sT[j][e] = dpT[j][e] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      uint32_t ak[4], av[4];
      ldsm_x4(smem_u32(sK) + swz(wk + (lane & 15), kk * 2 + (lane >> 4), RC), ak[0], ak[1], ak[2],
              ak[3]);
      ldsm_x4(smem_u32(sV) + swz(wk + (lane & 15), kk * 2 + (lane >> 4), RC), av[0], av[1], av[2],
              av[3]);
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        const int qrow = np * 16 + (lane & 7) + ((lane >> 4) << 3);
        const int ch = kk * 2 + ((lane >> 3) & 1);
        uint32_t b0, b1, b2, b3;
        ldsm_x4(sQ + swz(qrow, ch, RC), b0, b1, b2, b3);
        mma_bf16_16816(sT[2 * np], ak, b0, b1);
        mma_bf16_16816(sT[2 * np + 1], ak, b2, b3);
        ldsm_x4(sO + swz(qrow, ch, RC), b0, b1, b2, b3);
        mma_bf16_16816(dpT[2 * np], av, b0, b1);
        mma_bf16_16816(dpT[2 * np + 1], av, b2, b3);
      }
    }
    // ---- P^T and dS^T
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int c = c0 + wk + (lane >> 2) + ((e >> 1) << 3);
        const int rl = j * 8 + (lane & 3) * 2 + (e & 1);
        const int r = rq0 + rl;
        const bool vis = r < p.Lq && key_visible(p, r, c);
        const float pv = vis ? fast_exp2(fmaf(sT[j][e], p.scale_log2, -sL[st * 64 + rl])) : 0.f;
        sT[j][e] = pv;
        dpT[j][e] = pv * (dpT[j][e] - sDl[st * 64 + rl]);
      }
    // ---- dV += P^T dO ; dK += dS^T Q
#pragma unroll
    for (int kq = 0; kq < 4; ++kq) {
      uint32_t ap[4], as[4];
      ap[0] = pack_bf16(sT[2 * kq][0], sT[2 * kq][1]);
      ap[1] = pack_bf16(sT[2 * kq][2], sT[2 * kq][3]);
      ap[2] = pack_bf16(sT[2 * kq + 1][0], sT[2 * kq + 1][1]);
      ap[3] = pack_bf16(sT[2 * kq + 1][2], sT[2 * kq + 1][3]);
      as[0] = pack_bf16(dpT[2 * kq][0], dpT[2 * kq][1]);
      as[1] = pack_bf16(dpT[2 * kq][2], dpT[2 * kq][3]);
      as[2] = pack_bf16(dpT[2 * kq + 1][0], dpT[2 * kq + 1][1]);
      as[3] = pack_bf16(dpT[2 * kq + 1][2], dpT[2 * kq + 1][3]);
      const int qrow = kq * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
#pragma unroll
      for (int dp = 0; dp < D / 16; ++dp) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(sO + swz(qrow, dp * 2 + (lane >> 4), RC), b0, b1, b2, b3);
        mma_bf16_16816(dv[2 * dp], ap, b0, b1);
        mma_bf16_16816(dv[2 * dp + 1], ap, b2, b3);
        ldsm_x4_t(sQ + swz(qrow, dp * 2 + (lane >> 4), RC), b0, b1, b2, b3);
        mma_bf16_16816(dk[2 * dp], as, b0, b1);
        mma_bf16_16816(dk[2 * dp + 1], as, b2, b3);
      }
    }
    // ---- dS^T -> shared [key][query] (bf16)
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        const int row = wk + (lane >> 2) + hr * 8;
        const int col = j * 8 + (lane & 3) * 2;
        asm volatile("st.shared.b32 [%0], %1;\n" ::"r"(sS + swz(row, col >> 3, 8) + (col & 7) * 2),
                     "r"(pack_bf16(dpT[j][2 * hr], dpT[j][2 * hr + 1])));
      }
    __syncthreads();
    // ---- dQ (this warp: queries wk..wk+15 of the tile) += dS K over the 64 keys
    float* dqg = p.dq_acc + (q_row0 * p.Hq + h) * D;
#pragma unroll
    for (int dc = 0; dc < D / 32; ++dc) {
      float acc[4][4];
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        uint32_t a[4];
        ldsm_x4_t(sS + swz(kk * 16 + (lane & 7) + ((lane >> 4) << 3), warp * 2 + ((lane >> 3) & 1), 8),
                  a[0], a[1], a[2], a[3]);
        const int krow = kk * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
#pragma unroll
        for (int np = 0; np < 2; ++np) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(smem_u32(sK) + swz(krow, dc * 4 + np * 2 + (lane >> 4), RC), b0, b1, b2, b3);
          mma_bf16_16816(acc[2 * np], a, b0, b1);
          mma_bf16_16816(acc[2 * np + 1], a, b2, b3);
        }
      }
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        const int r = rq0 + wk + (lane >> 2) + hr * 8;
        if (r < p.Lq) {
          float* rowp = dqg + static_cast<long long>(r) * q_rs + dc * 32 + (lane & 3) * 2;
#pragma unroll
          for (int j = 0; j < 4; ++j)
            atomicAdd(reinterpret_cast<float2*>(rowp + j * 8),
                      make_float2(acc[j][2 * hr], acc[j][2 * hr + 1]));
        }
      }
    }
    __syncthreads();
  }
  cp_async_wait<0>();
  __syncthreads();

  // ---- dK (scaled), dV -> bf16 through shared memory (stage-0 Q / dO buffers)
#pragma unroll
  for (int j = 0; j < NDT; ++j)
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      const int row = wk + (lane >> 2) + hr * 8;
      const int col = j * 8 + (lane & 3) * 2;
      const uint32_t off = swz(row, col >> 3, RC) + (col & 7) * 2;
      asm volatile("st.shared.b32 [%0], %1;\n" ::"r"(sQ0 + off),
                   "r"(pack_bf16(dk[j][2 * hr] * p.scale, dk[j][2 * hr + 1] * p.scale)));
      asm volatile("st.shared.b32 [%0], %1;\n" ::"r"(sO0 + off),
                   "r"(pack_bf16(dv[j][2 * hr], dv[j][2 * hr + 1])));
    }
  __syncthreads();
  __nv_bfloat16* dkg = p.dk + (k_row0 * p.Hkv + hk) * D;
  __nv_bfloat16* dvg = p.dv + (k_row0 * p.Hkv + hk) * D;
  const uint8_t* sdk = smem + SM::Q_OFF;
  const uint8_t* sdv = smem + SM::DO_OFF;
  for (int i = tid; i < kBwdBN * RC; i += kBwdThreads) {
    const int row = i / RC, ch = i % RC, c = c0 + row;
    if (c < p.Lk) {
      const long long off = static_cast<long long>(c) * k_rs + ch * 8;
      *reinterpret_cast<uint4*>(dkg + off) = *reinterpret_cast<const uint4*>(sdk + swz(row, ch, RC));
      *reinterpret_cast<uint4*>(dvg + off) = *reinterpret_cast<const uint4*>(sdv + swz(row, ch, RC));
    }
  }
}

template <int D>
cudaError_t launch_bwd_d(const AttnParams& p, cudaStream_t stream) {
  const long long rows = static_cast<long long>(p.B) * p.Sq * p.Hq;
  bwd_pre_kernel<<<static_cast<unsigned>((rows + 7) / 8), 256, 0, stream>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int smem = BwdSmem<D>::TOTAL;
  e = cudaFuncSetAttribute(bwd_main_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const long long num_kt = (p.Lk + kBwdBN - 1) / kBwdBN;
  const long long blocks = num_kt * p.B * p.Hkv * p.groups;
  bwd_main_kernel<D><<<static_cast<unsigned>(blocks), kBwdThreads, smem, stream>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (p.mode == HD_INTRA && p.final_only && p.n > 1) {
    const long long kv_rows = static_cast<long long>(p.B) * p.S * p.Hkv;
    bwd_zero_unread_kv_kernel<<<static_cast<unsigned>((kv_rows + 7) / 8), 256, 0, stream>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  const long long n8 = rows * D / 8;
  bwd_dq_kernel<<<static_cast<unsigned>((n8 + 255) / 256), 256, 0, stream>>>(p, n8);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_bwd_mma(const AttnParams& p, cudaStream_t stream) {
  if (p.D == 64) return launch_bwd_d<64>(p, stream);
  if (p.D == 128) return launch_bwd_d<128>(p, stream);
  return cudaErrorInvalidValue;
}

}  // namespace hd
