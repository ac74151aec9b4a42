// attn_fwd_tc.cu - Stream-Factorized attention forward on the 5th-generation
// tensor cores (tcgen05 + TMEM + TMA), sm_100a.
//
// Computes, for every query row r of a problem (AttnParams, hd_common.cuh),
//   O_r = sum_c softmax_c(scale * q_r . k_c) v_c  over visible keys c, and LSE_r.
// Source: page "微信WeLM提出Hidden Decoding：大模型推理新范式" (tahou.com), section
// "规模化落地的工程优化" (intra-stream / cross-stream layers, KV-mirror) and
// section "隐式序列缩放的技术细节" step 2 (causal attention over the expanded
// sequence).
//
// One CTA = one 128-row query tile of one (batch, head, stream group).
//   warp 0      TMA producer: Q once, then K and V tiles of 128 keys into a
//               2-stage ring (128-byte swizzle). The 4-D tensor maps are
//               (d, head-or-stream*head, row, batch), so an INTRA stream is read
//               as a contiguous causal problem (row stride n*H*D), with no copy.
//   warp 1      allocates TMEM; lane 0 issues every tcgen05.mma:
//               S_i = Q K_i^T into one of two TMEM S buffers (M=128, N=128),
//               O += P_i V_i into the TMEM O accumulator (M=128, N=D, V read
//               MN-major straight from its TMA tile).
//   warps 4-7   softmax warpgroup, one query row per thread (= TMEM lane):
//               tcgen05.ld of the S row, mask on boundary tiles, online softmax
//               in base 2, P (bf16) into shared memory in the MMA's K-major
//               128-byte-swizzled layout. The running max is only raised when
//               a tile's max exceeds it by more than 2^8, so the O accumulator
//               is rescaled in TMEM rarely; the final 1/l and LSE make the
//               result exact either way.
// S_{i+1} runs on the tensor core while the softmax of tile i runs.
// Every mbarrier wait is bounded; on expiry the kernel records HD_ERR_TIMEOUT,
// every role leaves its loop, TMEM is freed and the kernel returns.
#include <cuda.h>

#include "hd_common.cuh"
#include "launch.h"
#include "tc_ptx.cuh"

namespace hd {

namespace {

constexpr int kBM = 128;  // query rows per CTA
constexpr int kBN = 128;  // keys per tile
constexpr int kThreads = 256;
constexpr int kSub = 128 * 128;  // bytes of one [128 rows][64 bf16] swizzled sub-tile
constexpr uint32_t kTmemCols = 512;

template <int D>
struct TcSmem {
  static constexpr int NSUB = D / 64;
  static constexpr int Q_BYTES = kBM * D * 2;
  static constexpr int KV_BYTES = kBN * D * 2;
  static constexpr int P_BYTES = kBM * kBN * 2;
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = Q_OFF + Q_BYTES;
  static constexpr int V_OFF = K_OFF + 2 * KV_BYTES;
  static constexpr int P_OFF = V_OFF + 2 * KV_BYTES;
  static constexpr int BAR_OFF = P_OFF + P_BYTES;
  // barriers: q_full, k_full[2], v_full[2], kv_empty[2], s_full[2], s_free[2], p_full, o_done
  static constexpr int NBAR = 13;
  static constexpr int SLOT_OFF = BAR_OFF + NBAR * 8;  // TMEM base address
  static constexpr int ABORT_OFF = SLOT_OFF + 4;
  // + alignment slack; at least 120 KB so that one CTA (and one 512-column
  // TMEM allocation) is resident per SM
  static constexpr int TOTAL = (ABORT_OFF + 4 + 1024) > 120 * 1024 ? (ABORT_OFF + 4 + 1024) : 120 * 1024;
};

enum { B_QF = 0, B_KF = 1, B_VF = 3, B_KE = 5, B_SF = 7, B_SE = 9, B_PF = 11, B_OD = 12 };

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_tc_kernel(const AttnParams p, const __grid_constant__ CUtensorMap tmQ,
                       const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                       const __grid_constant__ CUtensorMap tmO) {
  using SM = TcSmem<D>;
  constexpr int NSUB = SM::NSUB;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - smem_u32(smem_raw));
  const uint32_t sQ = sbase + SM::Q_OFF, sK = sbase + SM::K_OFF, sV = sbase + SM::V_OFF,
                 sP = sbase + SM::P_OFF;
  auto bar = [&](int i) { return sbase + SM::BAR_OFF + 8u * i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sgen + SM::ABORT_OFF);
  const uint32_t slot = sbase + SM::SLOT_OFF;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // A timeout recorded by an earlier CTA (or call) is sticky until the status
  // word is cleared: skip the work instead of waiting again.
  if (p.status && *reinterpret_cast<volatile int*>(p.status) == HD_ERR_TIMEOUT) return;

  // ---- problem of this CTA
  const int bhg = p.B * p.Hq * p.groups;
  const int num_qt = (p.Lq + kBM - 1) / kBM;
  const int qt = num_qt - 1 - static_cast<int>(blockIdx.x / bhg);  // heavy tiles first
  int y = static_cast<int>(blockIdx.x % bhg);
  const int grp = y % p.groups;
  y /= p.groups;
  const int h = y % p.Hq;
  const int b = y / p.Hq;
  const int hk = h / (p.Hq / p.Hkv);
  const bool intra = p.mode == HD_INTRA;
  const int jq = (intra && !p.final_only) ? grp * p.Hq + h : h;
  const int jk = intra ? (p.final_only ? p.n - 1 : grp) * p.Hkv + hk : hk;
  const int r0 = qt * kBM;
  const int r_last = min(r0 + kBM, p.Lq) - 1;
  const int kmax = min(p.Lk - 1, p.a * r_last + p.bb);
  const int kmin = max(0, p.a * r0 + p.bb - p.win + 1);
  const int kt_lo = kmin / kBN;
  const int nt = kmax / kBN - kt_lo + 1;

  if (tid == 0) {
    // softmax warps arrive once per warp (4); everything else arrives once
    for (int i = 0; i < SM::NBAR; ++i)
      tc::mbar_init(bar(i), (i == B_SE || i == B_SE + 1 || i == B_PF) ? 4 : 1);
    *abort_flag = 0;
    tc::fence_mbar_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(slot, kTmemCols);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sgen + SM::SLOT_OFF);
  const uint32_t tS = tmem, tO = tmem + 256;  // S buffers at columns 0 and 128, O at 256

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tc::tma_prefetch_desc(&tmQ);
      tc::tma_prefetch_desc(&tmK);
      tc::tma_prefetch_desc(&tmV);
      tc::mbar_expect_tx(bar(B_QF), SM::Q_BYTES);
#pragma unroll
      for (int s = 0; s < NSUB; ++s) tc::tma_load_4d(sQ + s * kSub, &tmQ, bar(B_QF), s * 64, jq, r0, b);
      for (int i = 0; i < nt; ++i) {
        const int st = i & 1;
        if (!tc::mbar_wait(bar(B_KE + st), ((i >> 1) & 1) ^ 1, abort_flag, p.status)) break;
        const int c0 = (kt_lo + i) * kBN;
        tc::mbar_expect_tx(bar(B_KF + st), SM::KV_BYTES);
#pragma unroll
        for (int s = 0; s < NSUB; ++s)
          tc::tma_load_4d(sK + st * SM::KV_BYTES + s * kSub, &tmK, bar(B_KF + st), s * 64, jk, c0, b);
        tc::mbar_expect_tx(bar(B_VF + st), SM::KV_BYTES);
#pragma unroll
        for (int s = 0; s < NSUB; ++s)
          tc::tma_load_4d(sV + st * SM::KV_BYTES + s * kSub, &tmV, bar(B_VF + st), s * 64, jk, c0, b);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = tc::idesc_bf16_f32(kBM, kBN, 0, 0);
      constexpr uint32_t idO = tc::idesc_bf16_f32(kBM, D, 0, 1);
      auto issue_S = [&](int buf, int st) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kSub + (kk & 3) * 32;
          tc::mma_ss(tS + buf * 128, tc::smem_desc_sw128(sQ + off, 16, 1024),
                     tc::smem_desc_sw128(sK + st * SM::KV_BYTES + off, 16, 1024), idS, kk > 0);
        }
      };
      bool ok = tc::mbar_wait(bar(B_QF), 0, abort_flag, p.status) &&
                tc::mbar_wait(bar(B_KF), 0, abort_flag, p.status);
      if (ok) {
        tc::tc_fence_after();
        issue_S(0, 0);
        tc::mma_commit(bar(B_SF));
      }
      for (int i = 0; ok && i < nt; ++i) {
        const int st = i & 1;
        if (i + 1 < nt) {
          const int s1 = (i + 1) & 1;
          ok = tc::mbar_wait(bar(B_KF + s1), ((i + 1) >> 1) & 1, abort_flag, p.status);
          if (ok && i + 1 >= 2)
            ok = tc::mbar_wait(bar(B_SE + s1), (((i + 1) >> 1) - 1) & 1, abort_flag, p.status);
          if (!ok) break;
          tc::tc_fence_after();
          issue_S(s1, s1);
          tc::mma_commit(bar(B_SF + s1));
        }
        ok = tc::mbar_wait(bar(B_PF), i & 1, abort_flag, p.status) &&
             tc::mbar_wait(bar(B_VF + st), (i >> 1) & 1, abort_flag, p.status);
        if (!ok) break;
        tc::tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
          const uint64_t ad = tc::smem_desc_sw128(sP + (kk >> 2) * kSub + (kk & 3) * 32, 16, 1024);
          const uint64_t bd = tc::smem_desc_sw128(sV + st * SM::KV_BYTES + kk * 2048, kSub, 1024);
          tc::mma_ss(tO, ad, bd, idO, (i > 0 || kk > 0) ? 1u : 0u);
        }
        tc::mma_commit(bar(B_OD));
        tc::mma_commit(bar(B_KE + st));
      }
    }
  } else if (warp >= 4) {
    // --------------------------------------------------------- softmax warpgroup
    const int row = tid - 128;
    const int r = r0 + row;
    const uint32_t tq = static_cast<uint32_t>((warp - 4) * 32) << 16;
    const int hi = p.a * r + p.bb;
    const int lo = hi - p.win;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int i = 0; i < nt; ++i) {
      const int st = i & 1;
      if (!tc::mbar_wait(bar(B_SF + st), (i >> 1) & 1, abort_flag, p.status)) { ok = false; break; }
      tc::tc_fence_after();
      uint32_t sr[kBN];
#pragma unroll
      for (int c = 0; c < kBN / 32; ++c) tc::tmem_ld32(tS + tq + st * 128 + c * 32, sr + c * 32);
      tc::tmem_wait_ld();
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(bar(B_SE + st));
      float* s = reinterpret_cast<float*>(sr);
      const int c0 = (kt_lo + i) * kBN;
      const bool full = (c0 + kBN - 1 <= p.a * r0 + p.bb) &&
                        (c0 > p.a * r_last + p.bb - p.win) && (c0 + kBN <= p.Lk);
      if (!full) {
#pragma unroll
        for (int j = 0; j < kBN; ++j) {
          const int c = c0 + j;
          if (!(c <= hi && c > lo && c < p.Lk)) s[j] = -INFINITY;
        }
      }
      float mx = -INFINITY;
#pragma unroll
      for (int j = 0; j < kBN; ++j) mx = fmaxf(mx, s[j]);
      const float m_tile = mx * p.scale_log2;
      if (i > 0) {
        if (!tc::mbar_wait(bar(B_OD), (i - 1) & 1, abort_flag, p.status)) { ok = false; break; }
        tc::tc_fence_after();
      }
      const bool need = m_tile > m_run + 8.f;
      if (__any_sync(0xffffffffu, need)) {
        const float m_new = fmaxf(m_run, m_tile);
        const float alpha = (m_run == -INFINITY) ? 0.f : fast_exp2(m_run - m_new);
        if (i > 0) {
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tc::tmem_ld32(tO + tq + c * 32, o);
            tc::tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
            tc::tmem_st32(tO + tq + c * 32, o);
          }
          tc::tmem_wait_st();
        }
        l_run *= alpha;
        m_run = m_new;
      }
      const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
      // P row -> shared memory, K-major 128-byte swizzle: chunk k of 8 keys
#pragma unroll
      for (int k = 0; k < kBN / 8; ++k) {
        float pv[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          pv[e] = fast_exp2(fmaf(s[k * 8 + e], p.scale_log2, -m_use));
          l_run += pv[e];
        }
        const uint32_t addr = sP + (k >> 3) * kSub + row * 128 + (((k & 7) ^ (row & 7)) << 4);
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};\n" ::"r"(addr),
                     "r"(pack_bf16(pv[0], pv[1])), "r"(pack_bf16(pv[2], pv[3])),
                     "r"(pack_bf16(pv[4], pv[5])), "r"(pack_bf16(pv[6], pv[7]))
                     : "memory");
      }
      tc::fence_async_smem();
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(bar(B_PF));
    }
    if (ok && !*abort_flag) ok = tc::mbar_wait(bar(B_OD), (nt - 1) & 1, abort_flag, p.status);
    if (ok) {
      tc::tc_fence_after();
      const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
      // O row -> bf16 -> shared memory (the Q tile's space, same swizzled layout)
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tc::tmem_ld32(tO + tq + c * 32, o);
        tc::tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int d8 = c * 4 + k;  // chunk of 8 columns
          const float* f = reinterpret_cast<const float*>(o + k * 8);
          const uint32_t addr = sQ + (d8 >> 3) * kSub + row * 128 + (((d8 & 7) ^ (row & 7)) << 4);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};\n" ::"r"(addr),
                       "r"(pack_bf16(f[0] * inv, f[1] * inv)), "r"(pack_bf16(f[2] * inv, f[3] * inv)),
                       "r"(pack_bf16(f[4] * inv, f[5] * inv)), "r"(pack_bf16(f[6] * inv, f[7] * inv))
                       : "memory");
        }
      }
      if (r < p.Lq) {
        const long long li = (static_cast<long long>(b) * p.Hq + h) * p.Sq +
                             static_cast<long long>(grp) * p.qs_step +
                             static_cast<long long>(r) * p.q_rstride;
        p.lse[li] = (m_run + __log2f(l_run)) * 0.69314718055994530942f;
      }
      tc::fence_async_smem();
    }
    asm volatile("bar.sync 1, 128;\n" ::: "memory");
    if (row == 0 && ok && !*abort_flag) {
#pragma unroll
      for (int s = 0; s < NSUB; ++s) tc::tma_store_4d(&tmO, sQ + s * kSub, s * 64, jq, r0, b);
      tc::tma_store_commit_and_wait();
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

// ----------------------------------------------------------------- host side
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// bf16 tensor viewed as (d, j, row, batch) with a box of 64 x 1 x 128 x 1.
bool make_map(CUtensorMap* map, const void* base, int D, long long J, long long R, long long B,
              long long stride_j, long long stride_r, long long stride_b) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(J),
                              static_cast<cuuint64_t>(R), static_cast<cuuint64_t>(B)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(stride_j * 2),
                                 static_cast<cuuint64_t>(stride_r * 2),
                                 static_cast<cuuint64_t>(stride_b * 2)};
  const cuuint32_t box[4] = {64, 1, 128, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
cudaError_t launch_tc_d(const AttnParams& p, cudaStream_t stream) {
  const long long S = p.S, L = p.L, n = p.n, Hq = p.Hq, Hkv = p.Hkv, B = p.B;
  CUtensorMap mq, mk, mv, mo;
  const bool intra = p.mode == HD_INTRA;
  bool ok;
  if (intra && !p.final_only) {
    ok = make_map(&mq, p.q, D, n * Hq, L, B, D, n * Hq * D, S * Hq * D) &&
         make_map(&mo, p.o, D, n * Hq, L, B, D, n * Hq * D, S * Hq * D);
  } else {
    const long long Rq = p.final_only ? L : S;
    ok = make_map(&mq, p.q, D, Hq, Rq, B, D, Hq * D, Rq * Hq * D) &&
         make_map(&mo, p.o, D, Hq, Rq, B, D, Hq * D, Rq * Hq * D);
  }
  if (intra) {
    ok = ok && make_map(&mk, p.k, D, n * Hkv, L, B, D, n * Hkv * D, S * Hkv * D) &&
         make_map(&mv, p.v, D, n * Hkv, L, B, D, n * Hkv * D, S * Hkv * D);
  } else {
    ok = ok && make_map(&mk, p.k, D, Hkv, S, B, D, Hkv * D, S * Hkv * D) &&
         make_map(&mv, p.v, D, Hkv, S, B, D, Hkv * D, S * Hkv * D);
  }
  if (!ok) return cudaErrorInvalidValue;
  const int smem = TcSmem<D>::TOTAL;
  cudaError_t e = cudaFuncSetAttribute(attn_fwd_tc_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const long long blocks = static_cast<long long>((p.Lq + kBM - 1) / kBM) * p.B * p.Hq * p.groups;
  attn_fwd_tc_kernel<D><<<static_cast<unsigned>(blocks), kThreads, smem, stream>>>(p, mq, mk, mv, mo);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_fwd_tc(const AttnParams& p, cudaStream_t stream) {
  if (p.D == 64) return launch_tc_d<64>(p, stream);
  if (p.D == 128) return launch_tc_d<128>(p, stream);
  return cudaErrorInvalidValue;
}

}  // namespace hd
