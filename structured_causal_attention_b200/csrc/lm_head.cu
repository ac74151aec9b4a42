// lm_head.cu - final-stream readout and the fused LM-head cross-entropy.
//
// Page "微信WeLM提出Hidden Decoding：大模型推理新范式" (tahou.com), section
// "隐式序列缩放的技术细节", step 3: in training only the last stream of every
// token carries the next-token loss. With hidden states X [B, n*L, d] of the
// expanded sequence, token t of sequence b is read out at position t*n + n-1:
//   h_r = X[b, t*n + n-1, :],   r = b*L + t,
//   loss_r = logsumexp_v (h_r . W_v) - h_r . W_label(r)   (W [V, d], no bias).
//
// lm_head_ce_kernel: a persistent tcgen05 GEMM of the final-stream rows against
// the LM head whose epilogue reduces each 256-wide vocabulary tile of a row to
// (max, sum of exp) in base 2, plus the label's logit when it falls in the
// tile: the [rows, V] logits never reach global memory. The readout is free:
// the rows' tensor map has row stride n*d, so the TMA reads the final stream
// in place.
//   unit      2 row tiles of 128 (A0, A1) x one vocabulary tile of 256 (B):
//             both MMA chains share every B tile (M=128, N=256, K=16 each).
//   warp 0    TMA producer: per 64-wide K block, A0, A1 and B into a 3-stage
//             ring of 64 KB stages (128-byte swizzle, K-major).
//   warp 1    allocates TMEM (512 columns: D0 at 0, D1 at 256); lane 0 issues
//             the MMAs and commits stage releases and the unit's accumulators.
//   warps 2-5 epilogue: one row of D0 and one of D1 per thread (TMEM lane =
//             row), 32-column tcgen05.ld chunks, online max / sum of exp2.
// Units are ordered in groups of kGroupRows row pairs x all vocabulary tiles,
// so the CTAs running at once share their row tiles and vocabulary tiles in L2.
// lm_head_combine_kernel merges the per-tile partials of a row into its
// logsumexp and loss.
// Every mbarrier wait is bounded; on expiry the kernel records HD_ERR_TIMEOUT,
// every role leaves its loop, TMEM is freed and the kernel returns.
#include <cuda.h>

#include "hd_common.cuh"
#include "launch.h"
#include "tc_ptx.cuh"

namespace hd {

namespace {

constexpr int kLR = 128;        // rows per A tile
constexpr int kLV = 256;        // vocabulary entries per unit
constexpr int kLK = 64;         // K elements per stage (128-byte rows)
constexpr int kLStages = 3;
constexpr int kLThreads = 192;  // 6 warps
constexpr int kGroupRows = 8;   // row pairs per raster group
constexpr uint32_t kLTmemCols = 512;
constexpr int kABytes = kLR * kLK * 2;  // 16 KB
constexpr int kBBytes = kLV * kLK * 2;  // 32 KB
constexpr int kStageBytes = 2 * kABytes + kBBytes;
enum { LB_FULL = 0, LB_EMPTY = kLStages, LB_ACC_FULL = 2 * kLStages, LB_ACC_EMPTY, LB_N };
constexpr int kBarOff = kLStages * kStageBytes;
constexpr int kSlotOff = kBarOff + LB_N * 8;
constexpr int kAbortOff = kSlotOff + 4;
constexpr int kLSmem = kAbortOff + 4 + 1024;  // + alignment slack for the 1024-B swizzle atoms
static_assert(kLSmem <= 232448, "shared memory");

constexpr float kLog2e = 1.4426950408889634074f;
constexpr float kLn2f = 0.69314718055994530942f;

struct LmUnit {
  int rb, vt;
};

__device__ __forceinline__ LmUnit unit_of(long long u, int nrb, int nvt) {
  const long long per_group = static_cast<long long>(kGroupRows) * nvt;
  const int grp = static_cast<int>(u / per_group);
  const int within = static_cast<int>(u % per_group);
  const int rows_here = min(kGroupRows, nrb - grp * kGroupRows);
  return {grp * kGroupRows + within % rows_here, within / rows_here};
}

// x[k] for a thread-dependent k in [0, 32), as a tree of selects on the bits
// of k (an indexed read would put x in local memory).
__device__ __forceinline__ float select32(const uint32_t* x, int k) {
  uint32_t v[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) v[j] = (k & 16) ? x[j + 16] : x[j];
#pragma unroll
  for (int j = 0; j < 8; ++j) v[j] = (k & 8) ? v[j + 8] : v[j];
#pragma unroll
  for (int j = 0; j < 4; ++j) v[j] = (k & 4) ? v[j + 4] : v[j];
#pragma unroll
  for (int j = 0; j < 2; ++j) v[j] = (k & 2) ? v[j + 2] : v[j];
  return __uint_as_float((k & 1) ? v[1] : v[0]);
}

// kGrad = false: the loss epilogue (per-tile max / sum of exp2, label logit).
// kGrad = true: the gradient epilogue, G[r, v] = 2^(logit log2 e - LSE_r log2 e)
// - [v == label_r] as bf16 into p.g (row stride p.g_ld), zero for rows without
// a target and for the padding columns v >= V.
template <bool kGrad>
__global__ void __launch_bounds__(kLThreads, 1)
    lm_head_ce_kernel(const LmHeadParams p, const __grid_constant__ CUtensorMap tmA,
                      const __grid_constant__ CUtensorMap tmW) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - smem_u32(smem_raw));
  auto bar = [&](int i) { return sbase + kBarOff + 8u * i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sgen + kAbortOff);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (p.status && *reinterpret_cast<volatile int*>(p.status) == HD_ERR_TIMEOUT) return;

  if (tid == 0) {
    for (int i = 0; i < LB_N; ++i) tc::mbar_init(bar(i), i == LB_ACC_EMPTY ? 4 : 1);
    *abort_flag = 0;
    tc::fence_mbar_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(sbase + kSlotOff, kLTmemCols);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sgen + kSlotOff);
  const int nkb = p.d / kLK;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tc::tma_prefetch_desc(&tmA);
      tc::tma_prefetch_desc(&tmW);
      int it = 0;
      bool ok = true;
      for (long long u = blockIdx.x; ok && u < p.units; u += gridDim.x) {
        const LmUnit w = unit_of(u, p.nrb, p.nvt);
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const int s = it % kLStages;
          if (!tc::mbar_wait(bar(LB_EMPTY + s), ((it / kLStages) & 1) ^ 1, abort_flag, p.status)) {
            ok = false;
            break;
          }
          const uint32_t dst = sbase + s * kStageBytes;
          tc::mbar_expect_tx(bar(LB_FULL + s), kStageBytes);
          tc::tma_load_2d(dst, &tmA, bar(LB_FULL + s), kb * kLK, w.rb * 2 * kLR);
          tc::tma_load_2d(dst + kABytes, &tmA, bar(LB_FULL + s), kb * kLK, w.rb * 2 * kLR + kLR);
          tc::tma_load_2d(dst + 2 * kABytes, &tmW, bar(LB_FULL + s), kb * kLK, w.vt * kLV);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = tc::idesc_bf16_f32(kLR, kLV, 0, 0);
      int it = 0, ui = 0;
      bool ok = true;
      for (long long u = blockIdx.x; ok && u < p.units; u += gridDim.x, ++ui) {
        // the epilogue must have read the previous unit's accumulators
        if (ui > 0 && !tc::mbar_wait(bar(LB_ACC_EMPTY), (ui - 1) & 1, abort_flag, p.status)) break;
        tc::tc_fence_after();
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const int s = it % kLStages;
          if (!tc::mbar_wait(bar(LB_FULL + s), (it / kLStages) & 1, abort_flag, p.status)) {
            ok = false;
            break;
          }
          tc::tc_fence_after();
          const uint32_t a0 = sbase + s * kStageBytes, a1 = a0 + kABytes, b0 = a0 + 2 * kABytes;
#pragma unroll
          for (int kk = 0; kk < kLK / 16; ++kk) {
            const uint64_t bd = tc::smem_desc_sw128(b0 + kk * 32, 16, 1024);
            const uint32_t acc = (kb > 0 || kk > 0) ? 1u : 0u;
            tc::mma_ss(tmem, tc::smem_desc_sw128(a0 + kk * 32, 16, 1024), bd, idesc, acc);
            tc::mma_ss(tmem + kLV, tc::smem_desc_sw128(a1 + kk * 32, 16, 1024), bd, idesc, acc);
          }
          tc::mma_commit(bar(LB_EMPTY + s));
        }
        if (ok) tc::mma_commit(bar(LB_ACC_FULL));
      }
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    const int quarter = warp & 3;  // TMEM lanes 32*quarter .. +31
    const uint32_t tq = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    int ui = 0;
    for (long long u = blockIdx.x; u < p.units; u += gridDim.x, ++ui) {
      const LmUnit w = unit_of(u, p.nrb, p.nvt);
      const int v0 = w.vt * kLV;
      int row[2], lab[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        row[h] = w.rb * 2 * kLR + h * kLR + quarter * 32 + lane;
        lab[h] = row[h] < p.R ? __ldg(p.labels + row[h]) : -1;
      }
      float lse2[2];
      if constexpr (kGrad) {
#pragma unroll
        for (int h = 0; h < 2; ++h) lse2[h] = row[h] < p.R ? __ldg(p.lse_in + row[h]) * kLog2e : 0.f;
      }
      if (!tc::mbar_wait_warp(bar(LB_ACC_FULL), ui & 1, abort_flag, p.status)) break;
      tc::tc_fence_after();
      if constexpr (kGrad) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const bool live = row[h] < p.R && lab[h] >= 0 && lab[h] < p.V;
          __nv_bfloat16* grow = p.g + static_cast<long long>(row[h]) * p.g_ld + v0;
          for (int c = 0; c < kLV / 32; ++c) {
            uint32_t x[32];
            tc::tmem_ld32(tq + h * kLV + c * 32, x);
            tc::tmem_wait_ld();
            uint32_t pk[16];
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
              const int v = v0 + c * 32 + j;
              float g0 = fast_exp2(fmaf(__uint_as_float(x[j]), kLog2e, -lse2[h])) - (v == lab[h] ? 1.f : 0.f);
              float g1 = fast_exp2(fmaf(__uint_as_float(x[j + 1]), kLog2e, -lse2[h])) -
                         (v + 1 == lab[h] ? 1.f : 0.f);
              g0 = (live && v < p.V) ? g0 : 0.f;
              g1 = (live && v + 1 < p.V) ? g1 : 0.f;
              pk[j >> 1] = pack_bf16(g0, g1);
            }
            if (row[h] < p.R &&
                in_bounds(static_cast<long long>(row[h]) * p.g_ld + v0 + c * 32, 32, p.R * p.g_ld, p.status)) {
              uint4* dst = reinterpret_cast<uint4*>(grow + c * 32);
#pragma unroll
              for (int q4 = 0; q4 < 4; ++q4)
                dst[q4] = make_uint4(pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]);
            }
          }
        }
      } else {
        const int nchunk = min(kLV, p.V - v0 + 31) / 32;  // chunks with at least one entry < V
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          float m = -INFINITY, l = 0.f, picked = 0.f;
          const int lo = lab[h] - v0;  // label's column in this tile, if in [0, 256)
          for (int c = 0; c < nchunk; ++c) {
            uint32_t x[32];
            tc::tmem_ld32(tq + h * kLV + c * 32, x);
            tc::tmem_wait_ld();
            if (lo >= c * 32 && lo < c * 32 + 32) picked = select32(x, lo - c * 32);
            const int valid = min(32, p.V - (v0 + c * 32));  // >= 1
            float y[32];
            float mx = -INFINITY;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              y[j] = j < valid ? __uint_as_float(x[j]) * kLog2e : -INFINITY;
              mx = fmaxf(mx, y[j]);
            }
            const float mn = fmaxf(m, mx);
            float s = 0.f;
#pragma unroll
            for (int j = 0; j < 32; ++j) s += fast_exp2(y[j] - mn);
            l = l * fast_exp2(m - mn) + s;
            m = mn;
          }
          if (row[h] < p.R && in_bounds(static_cast<long long>(p.nvt + w.vt) * p.R + row[h], 1,
                                        2LL * p.nvt * p.R, p.status)) {
            p.part[static_cast<long long>(w.vt) * p.R + row[h]] = m;
            p.part[static_cast<long long>(p.nvt + w.vt) * p.R + row[h]] = l;
            if (lo >= 0 && lo < kLV) p.pick[row[h]] = picked;
          }
        }
      }
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(bar(LB_ACC_EMPTY));
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, kLTmemCols);
  }
}

// ---------------------------------------------------------------------------
// C[M, N] = scale * A[M, K] B[K, N] on the tensor cores (bf16 operands, fp32
// accumulation in TMEM): the two GEMMs of the LM-head gradient. Persistent;
// a unit is one 128 x 256 tile of C, units walked with the N tiles inner so
// the CTAs running at once share their A rows in L2.
//   A: K-major (row m of A contiguous) or, with kAmn, M-major (A stored as
//      A^T, i.e. row k contiguous over m). B: N-major (row k contiguous).
//   warp 0    TMA producer, 64-wide K blocks into a 4-stage ring
//   warp 1    TMEM (2 accumulators of 256 columns); lane 0 issues M128 N256
//             K16 MMAs (long enough that issue keeps up with the tensor cores)
//   warps 2-5 epilogue: a row per thread, tcgen05.ld, scale, 16-byte stores;
//             the other accumulator takes the next unit's MMAs meanwhile.
constexpr int kGM = 128, kGN = 256, kGK = 64, kGStages = 4, kGThreads = 192;
constexpr int kGABytes = kGM * kGK * 2;   // 16 KB
constexpr int kGBBytes = kGK * kGN * 2;   // 32 KB
constexpr int kGStageBytes = kGABytes + kGBBytes;
enum { GB_FULL = 0, GB_EMPTY = kGStages, GB_AF = 2 * kGStages, GB_AE = GB_AF + 2, GB_N = GB_AE + 2 };
constexpr int kGBarOff = kGStages * kGStageBytes;
constexpr int kGSlotOff = kGBarOff + GB_N * 8;
constexpr int kGAbortOff = kGSlotOff + 4;
constexpr int kGSmem = kGAbortOff + 4 + 1024;
static_assert(kGSmem <= 232448, "shared memory");

struct GemmArgs {
  void* c;         // [M, ldc] bf16, or fp32 when c_fp32
  long long ldc;
  int M, N, K, c_fp32;
  float scale;
  int ntn;         // N tiles
  long long units;
  int* status;
};

template <bool kAmn>
__global__ void __launch_bounds__(kGThreads, 1)
    gemm_tc_kernel(const GemmArgs p, const __grid_constant__ CUtensorMap tmA,
                   const __grid_constant__ CUtensorMap tmB) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - smem_u32(smem_raw));
  auto bar = [&](int i) { return sbase + kGBarOff + 8u * i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sgen + kGAbortOff);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (p.status && *reinterpret_cast<volatile int*>(p.status) == HD_ERR_TIMEOUT) return;
  if (tid == 0) {
    for (int i = 0; i < GB_N; ++i) tc::mbar_init(bar(i), (i == GB_AE || i == GB_AE + 1) ? 4 : 1);
    *abort_flag = 0;
    tc::fence_mbar_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(sbase + kGSlotOff, 512);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sgen + kGSlotOff);
  const int nkb = (p.K + kGK - 1) / kGK;

  if (warp == 0) {
    if (lane == 0) {
      tc::tma_prefetch_desc(&tmA);
      tc::tma_prefetch_desc(&tmB);
      int it = 0;
      bool ok = true;
      for (long long u = blockIdx.x; ok && u < p.units; u += gridDim.x) {
        const int m0 = static_cast<int>(u / p.ntn) * kGM, n0 = static_cast<int>(u % p.ntn) * kGN;
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const int s = it % kGStages;
          if (!tc::mbar_wait(bar(GB_EMPTY + s), ((it / kGStages) & 1) ^ 1, abort_flag, p.status)) {
            ok = false;
            break;
          }
          const uint32_t sa = sbase + s * kGStageBytes, sb = sa + kGABytes;
          tc::mbar_expect_tx(bar(GB_FULL + s), kGStageBytes);
          if (kAmn) {
            tc::tma_load_2d(sa, &tmA, bar(GB_FULL + s), m0, kb * kGK);
            tc::tma_load_2d(sa + kGABytes / 2, &tmA, bar(GB_FULL + s), m0 + 64, kb * kGK);
          } else {
            tc::tma_load_2d(sa, &tmA, bar(GB_FULL + s), kb * kGK, m0);
          }
#pragma unroll
          for (int q4 = 0; q4 < kGN / 64; ++q4)
            tc::tma_load_2d(sb + q4 * (kGBBytes / 4), &tmB, bar(GB_FULL + s), n0 + 64 * q4, kb * kGK);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = tc::idesc_bf16_f32(kGM, kGN, kAmn ? 1 : 0, 1);
      int it = 0, ui = 0;
      bool ok = true;
      for (long long u = blockIdx.x; ok && u < p.units; u += gridDim.x, ++ui) {
        const int buf = ui & 1;
        // the epilogue has read this accumulator's previous unit
        if (ui >= 2 && !tc::mbar_wait(bar(GB_AE + buf), ((ui >> 1) - 1) & 1, abort_flag, p.status)) break;
        tc::tc_fence_after();
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const int s = it % kGStages;
          if (!tc::mbar_wait(bar(GB_FULL + s), (it / kGStages) & 1, abort_flag, p.status)) {
            ok = false;
            break;
          }
          tc::tc_fence_after();
          const uint32_t sa = sbase + s * kGStageBytes, sb = sa + kGABytes;
#pragma unroll
          for (int kk = 0; kk < kGK / 16; ++kk) {
            const uint64_t ad = kAmn ? tc::smem_desc_sw128(sa + kk * 2048, kGABytes / 2, 1024)
                                     : tc::smem_desc_sw128(sa + kk * 32, 16, 1024);
            const uint64_t bd = tc::smem_desc_sw128(sb + kk * 2048, kGBBytes / 4, 1024);
            tc::mma_ss(tmem + kGN * buf, ad, bd, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
          }
          tc::mma_commit(bar(GB_EMPTY + s));
        }
        if (ok) tc::mma_commit(bar(GB_AF + buf));
      }
    }
  } else {
    const int quarter = warp & 3;
    const uint32_t tq = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    int ui = 0;
    for (long long u = blockIdx.x; u < p.units; u += gridDim.x, ++ui) {
      const int buf = ui & 1;
      const int m0 = static_cast<int>(u / p.ntn) * kGM, n0 = static_cast<int>(u % p.ntn) * kGN;
      const int r = m0 + quarter * 32 + lane;
      if (!tc::mbar_wait_warp(bar(GB_AF + buf), (ui >> 1) & 1, abort_flag, p.status)) break;
      tc::tc_fence_after();
      for (int c = 0; c < kGN / 32; ++c) {
        uint32_t x[32];
        tc::tmem_ld32(tq + kGN * buf + c * 32, x);
        tc::tmem_wait_ld();
        const int col = n0 + c * 32;
        const long long ci = static_cast<long long>(r) * p.ldc + col;
        if (r < p.M && col < p.N && in_bounds(ci, 32, static_cast<long long>(p.M) * p.ldc, p.status)) {
          if (p.c_fp32) {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.c) + ci);
#pragma unroll
            for (int q4 = 0; q4 < 8; ++q4)
              dst[q4] = make_float4(__uint_as_float(x[4 * q4]) * p.scale, __uint_as_float(x[4 * q4 + 1]) * p.scale,
                                    __uint_as_float(x[4 * q4 + 2]) * p.scale, __uint_as_float(x[4 * q4 + 3]) * p.scale);
          } else {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.c) + ci);
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
              const float* f = reinterpret_cast<const float*>(x + 8 * q4);
              dst[q4] = make_uint4(pack_bf16(f[0] * p.scale, f[1] * p.scale), pack_bf16(f[2] * p.scale, f[3] * p.scale),
                                   pack_bf16(f[4] * p.scale, f[5] * p.scale), pack_bf16(f[6] * p.scale, f[7] * p.scale));
            }
          }
        }
      }
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(bar(GB_AE + buf));
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, 512);
  }
}

// One thread per row: merge the vocabulary tiles' (max, sum) partials.
__global__ void lm_head_combine_kernel(const LmHeadParams p) {
  const long long r = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (r >= p.R) return;
  float mx = -INFINITY;
  for (int t = 0; t < p.nvt; ++t) mx = fmaxf(mx, p.part[static_cast<long long>(t) * p.R + r]);
  float l = 0.f;
  for (int t = 0; t < p.nvt; ++t)
    l += p.part[static_cast<long long>(p.nvt + t) * p.R + r] *
         fast_exp2(p.part[static_cast<long long>(t) * p.R + r] - mx);
  const float lse = (mx + __log2f(l)) * kLn2f;
  const int label = __ldg(p.labels + r);
  float loss = 0.f;
  if (label >= p.V) {
    record_status(p.status, HD_ERR_DEVICE_INDEX);
  } else if (label >= 0) {
    loss = lse - p.pick[r];
  }
  p.loss[r] = loss;
  if (p.lse) p.lse[r] = lse;
}

// out[b, t, :] = x[b, t*n + n-1, :]: one warp per output row, 16-byte vectors.
__global__ void __launch_bounds__(256) final_readout_kernel(const uint8_t* __restrict__ x,
                                                            uint8_t* __restrict__ out, long long rows,
                                                            int n, long long row_bytes, int* status) {
  const int lane = threadIdx.x & 31;
  const long long warps = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
  const long long nvec = row_bytes / 16;
  for (long long r = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
       r < rows; r += warps) {
    if (!in_bounds((r * n + n - 1) * row_bytes, row_bytes, rows * n * row_bytes, status) ||
        !in_bounds(r * row_bytes, row_bytes, rows * row_bytes, status))
      continue;
    const uint4* src = reinterpret_cast<const uint4*>(x + (r * n + n - 1) * row_bytes);
    uint4* dst = reinterpret_cast<uint4*>(out + r * row_bytes);
    long long i = lane;
    for (; i + 96 < nvec; i += 128) {
      const uint4 a = __ldcs(src + i), b = __ldcs(src + i + 32), c = __ldcs(src + i + 64),
                  e = __ldcs(src + i + 96);
      dst[i] = a;
      dst[i + 32] = b;
      dst[i + 64] = c;
      dst[i + 96] = e;
    }
    for (; i < nvec; i += 32) dst[i] = __ldcs(src + i);
  }
}

// 2-D bf16 map (d, rows) with a row stride of `row_stride` elements and a
// box of 64 x box_rows, 128-byte swizzle.
bool make_map_2d(CUtensorMap* map, const void* base, long long d, long long rows,
                 long long row_stride, int box_rows) {
  using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                     const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                     const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                     CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return false;
    fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(row_stride * 2)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kLK), static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

size_t lm_head_workspace_bytes(long long R, int V) {
  const long long nvt = (V + kLV - 1) / kLV;
  const size_t part = static_cast<size_t>(2 * nvt * R) * 4;
  return ((part + 255) & ~static_cast<size_t>(255)) + ((static_cast<size_t>(R) * 4 + 255) & ~static_cast<size_t>(255));
}

cudaError_t launch_lm_head_ce(LmHeadParams p, const void* x, const void* w, int n, int num_sms,
                              cudaStream_t stream) {
  // rows r = b*L + t live at x + (r*n + n-1)*d: base shifted by (n-1)*d, row stride n*d
  const __nv_bfloat16* a_base = static_cast<const __nv_bfloat16*>(x) + static_cast<long long>(n - 1) * p.d;
  CUtensorMap ma, mw;
  if (!make_map_2d(&ma, a_base, p.d, p.R, static_cast<long long>(n) * p.d, kLR) ||
      !make_map_2d(&mw, w, p.d, p.V, p.d, kLV))
    return cudaErrorInvalidValue;
  p.nrb = static_cast<int>((p.R + 2 * kLR - 1) / (2 * kLR));
  p.nvt = (p.V + kLV - 1) / kLV;
  p.units = static_cast<long long>(p.nrb) * p.nvt;
  cudaError_t e = cudaFuncSetAttribute(lm_head_ce_kernel<false>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, kLSmem);
  if (e != cudaSuccess) return e;
  const long long grid = p.units < num_sms ? p.units : num_sms;
  lm_head_ce_kernel<false><<<static_cast<unsigned>(grid), kLThreads, kLSmem, stream>>>(p, ma, mw);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  lm_head_combine_kernel<<<static_cast<unsigned>((p.R + 255) / 256), 256, 0, stream>>>(p);
  return cudaGetLastError();
}

size_t lm_head_grad_workspace_bytes(long long R, int V) {
  const long long vp = (V + kLV - 1) / kLV * kLV;
  return (static_cast<size_t>(R * vp) * 2 + 255) & ~static_cast<size_t>(255);
}

namespace {

template <bool kAmn>
cudaError_t launch_gemm(const CUtensorMap& ma, const CUtensorMap& mb, GemmArgs a, int num_sms,
                        cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel<kAmn>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kGSmem);
  if (e != cudaSuccess) return e;
  const long long grid = a.units < num_sms ? a.units : num_sms;
  gemm_tc_kernel<kAmn><<<static_cast<unsigned>(grid), kGThreads, kGSmem, stream>>>(a, ma, mb);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_lm_head_ce_bwd(LmHeadParams p, const void* x, const void* w, int n, float scale,
                                  void* dh, float* dw, int num_sms, cudaStream_t stream) {
  const __nv_bfloat16* h_base = static_cast<const __nv_bfloat16*>(x) + static_cast<long long>(n - 1) * p.d;
  const long long hstride = static_cast<long long>(n) * p.d;
  // 1. G = softmax(logits) - onehot, bf16 [R, g_ld]
  CUtensorMap ma, mw;
  if (!make_map_2d(&ma, h_base, p.d, p.R, hstride, kLR) || !make_map_2d(&mw, w, p.d, p.V, p.d, kLV))
    return cudaErrorInvalidValue;
  p.nrb = static_cast<int>((p.R + 2 * kLR - 1) / (2 * kLR));
  p.nvt = (p.V + kLV - 1) / kLV;
  p.units = static_cast<long long>(p.nrb) * p.nvt;
  p.g_ld = static_cast<long long>(p.nvt) * kLV;
  cudaError_t e = cudaFuncSetAttribute(lm_head_ce_kernel<true>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, kLSmem);
  if (e != cudaSuccess) return e;
  long long grid = p.units < num_sms ? p.units : num_sms;
  lm_head_ce_kernel<true><<<static_cast<unsigned>(grid), kLThreads, kLSmem, stream>>>(p, ma, mw);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int ntn = (p.d + kGN - 1) / kGN;
  // 2. dh = scale * G W: A = G (K-major over the vocabulary), B = W (rows = vocabulary)
  {
    CUtensorMap ga, gb;
    if (!make_map_2d(&ga, p.g, p.g_ld, p.R, p.g_ld, kGM) || !make_map_2d(&gb, w, p.d, p.V, p.d, kGK))
      return cudaErrorInvalidValue;
    GemmArgs a{};
    a.c = dh;
    a.ldc = p.d;
    a.M = static_cast<int>(p.R);
    a.N = p.d;
    a.K = static_cast<int>(p.g_ld);
    a.c_fp32 = 0;
    a.scale = scale;
    a.ntn = ntn;
    a.units = (p.R + kGM - 1) / kGM * ntn;
    a.status = p.status;
    e = launch_gemm<false>(ga, gb, a, num_sms, stream);
    if (e != cudaSuccess) return e;
  }
  // 3. dW = scale * G^T h: A = G read vocabulary-major, B = the final-stream rows in place
  {
    CUtensorMap ga, gb;
    if (!make_map_2d(&ga, p.g, p.g_ld, p.R, p.g_ld, kGK) || !make_map_2d(&gb, h_base, p.d, p.R, hstride, kGK))
      return cudaErrorInvalidValue;
    GemmArgs a{};
    a.c = dw;
    a.ldc = p.d;
    a.M = p.V;
    a.N = p.d;
    a.K = static_cast<int>(p.R);
    a.c_fp32 = 1;
    a.scale = scale;
    a.ntn = ntn;
    a.units = static_cast<long long>((p.V + kGM - 1) / kGM) * ntn;
    a.status = p.status;
    e = launch_gemm<true>(ga, gb, a, num_sms, stream);
  }
  return e;
}

cudaError_t launch_final_readout(const void* x, void* out, long long rows, int n,
                                 long long row_bytes, int sms, int* status, cudaStream_t stream) {
  long long blocks = (rows + 7) / 8;
  const long long cap = static_cast<long long>(sms) * 16;  // grid-stride beyond 16 blocks per SM
  if (blocks > cap) blocks = cap;
  final_readout_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
      static_cast<const uint8_t*>(x), static_cast<uint8_t*>(out), rows, n, row_bytes, status);
  return cudaGetLastError();
}

}  // namespace hd
