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
// One CTA = one 128-row query tile of one (batch, head, stream group); two CTAs
// share an SM (256 TMEM columns and under 100 KB of shared memory each), so one
// CTA's tensor-core work runs while the other's softmax, start-up or output
// store does, and the two chains never wait on each other.
//   warps 0-3   softmax, one row per thread (= TMEM lane): tcgen05.ld of the S
//               row, mask on boundary tiles, online softmax in base 2, P as
//               bf16 pairs written back into the upper S columns of TMEM
//               (tcgen05.st). The running max is only raised when a tile's
//               max exceeds it by more than 2^8, so the O accumulator is
//               rescaled in TMEM rarely; the final 1/l and LSE make the result
//               exact either way. The row's scores are read from TMEM once and
//               kept in registers. Then the output: O/l as bf16 through the Q
//               tile's shared memory to a TMA store, and the LSE.
//   warp 4      TMA producer: the Q tile once, then K and V tiles of 128 keys
//               (128-byte swizzle), one buffer each: K(j+1) streams in while
//               S(j) is exponentiated, V(j+1) once PV(j) has read V(j). The 4-D
//               tensor maps are (d, head-or-stream*head, row, batch), so an
//               INTRA stream is read as a contiguous causal problem (row stride
//               n*H*D), with no copy.
//   warp 5      allocates TMEM ([S/P 128 columns | O D columns]) and walks the
//               MMA loop as a whole warp (warp-uniform operands), one elected
//               lane issuing every tcgen05.mma:
//               S = Q K^T (M=128, N=128, both operands from shared memory);
//               O += P V (M=128, N=D, P from TMEM, V MN-major from its TMA tile),
//               issued in two halves of 64 keys: the softmax signals P of keys
//               64-127 before it exponentiates keys 0-63, so half of PV runs
//               under the rest of the softmax. S(j+1) follows PV(j).
// MMAs from one thread execute in order, so when S(j) is complete, PV(j-1)
// (issued before it) has finished reading P and updating O: the softmax may
// then rescale O and overwrite P without another wait.
// Every mbarrier wait is bounded; on expiry the kernel records HD_ERR_TIMEOUT,
// every role leaves its loop, TMEM is freed and the kernel returns.
#include <cuda.h>

#include "hd_common.cuh"
#include "launch.h"
#include "tc_ptx.cuh"

namespace hd {

namespace {

constexpr int kBM = 128;        // query rows per CTA
constexpr int kBN = 128;        // keys per K/V tile
constexpr int kThreads = 192;   // warps 0-3 softmax, 4 TMA producer, 5 MMA issuer
constexpr int kSub = 128 * 128;  // bytes of one [128 rows][64 bf16] swizzled sub-tile
constexpr uint32_t kTmemCols = 256;
constexpr float kRescaleLog2 = 8.f;  // raise the running max only past 2^8

template <int D>
struct TcSmem {
  static constexpr int NSUB = D / 64;
  static constexpr int Q_BYTES = kBM * D * 2;
  static constexpr int KV_BYTES = kBN * D * 2;
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = Q_OFF + Q_BYTES;
  static constexpr int V_OFF = K_OFF + KV_BYTES;
  static constexpr int BAR_OFF = V_OFF + KV_BYTES;
  // q_full, k_full, v_full, k_empty, v_empty, s_full, p_hi, p_lo, o_final
  static constexpr int NBAR = 9;
  static constexpr int SLOT_OFF = BAR_OFF + NBAR * 8;
  static constexpr int ABORT_OFF = SLOT_OFF + 4;
  static constexpr int USED = ABORT_OFF + 4 + 1024;
  // at least 80 KB, so that at most two CTAs (2 x 256 TMEM columns) share an SM
  static constexpr int TOTAL = USED > 80 * 1024 ? USED : 80 * 1024;
};

// p_hi: P of keys 64-127 written; p_lo: P of keys 0-63 written
enum { B_QF = 0, B_KF = 1, B_VF = 2, B_KE = 3, B_VE = 4, B_SF = 5, B_PA = 6, B_PB = 7, B_OF = 8 };

// Grid order, heaviest query tiles first. Query-tile-major order balances
// short problems. For long full-causal ones (no window, one stream group, at
// least 128 query tiles) it spreads the CTAs running at once over every KV
// head, so each head's K/V tiles are read by CTAs far apart in time and come
// back from DRAM (about 200 GB of reads for one forward at 131072 positions,
// whose algorithmic bytes are 2.7 GB). Those problems take a KV-head-major
// order instead, and inside one KV head the heads of its group at each query
// tile: 3.2 GB of reads at an L2 hit rate of 99 %, and 4 % less time at the
// power cap.
__host__ __device__ __forceinline__ bool fwd_kv_major(const AttnParams& p, int num_qt) {
  return p.win >= p.Lk && p.groups == 1 && num_qt >= 128;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 2)
    attn_fwd_tc_kernel(const AttnParams p, const __grid_constant__ CUtensorMap tmQ,
                       const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                       const __grid_constant__ CUtensorMap tmO) {
  using SM = TcSmem<D>;
  constexpr int NSUB = SM::NSUB;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - smem_u32(smem_raw));
  const uint32_t sQ = sbase + SM::Q_OFF, sK = sbase + SM::K_OFF, sV = sbase + SM::V_OFF;
  auto bar = [&](int i) { return sbase + SM::BAR_OFF + 8u * i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sgen + SM::ABORT_OFF);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (p.status && *reinterpret_cast<volatile int*>(p.status) == HD_ERR_TIMEOUT) return;

  const int num_qt = (p.Lq + kBM - 1) / kBM;
  const int g = p.Hq / p.Hkv;
  int b, grp, h, qt;
  if (fwd_kv_major(p, num_qt)) {
    const int per_kv = num_qt * g;
    const int bk = static_cast<int>(blockIdx.x / per_kv);
    const int rem = static_cast<int>(blockIdx.x % per_kv);
    qt = num_qt - 1 - rem / g;
    grp = 0;
    b = bk / p.Hkv;
    h = (bk % p.Hkv) * g + rem % g;
  } else {
    const int bhg = p.B * p.Hq * p.groups;
    qt = num_qt - 1 - static_cast<int>(blockIdx.x / bhg);  // heavy tiles first
    int y = static_cast<int>(blockIdx.x % bhg);
    grp = y % p.groups;
    y /= p.groups;
    h = y % p.Hq;
    b = y / p.Hq;
  }
  const int r0 = qt * kBM;  // first query row of the tile
  const int hk = h / g;
  const bool intra = p.mode == HD_INTRA;
  const int jq = (intra && !p.final_only) ? grp * p.Hq + h : h;
  const int jk = intra ? (p.final_only ? p.n - 1 : grp) * p.Hkv + hk : hk;
  const int rq_last = min(r0 + kBM, p.Lq) - 1;
  // key tiles [kt_lo, kt_hi] hold every key some row of the tile sees
  const int kt_lo = max(0, p.a * r0 + p.bb - p.win + 1) / kBN;
  const int kt_hi = min(p.Lk - 1, p.a * rq_last + p.bb) / kBN;
  const int nkv = kt_hi - kt_lo + 1;

  if (tid == 0) {
    for (int i = 0; i < SM::NBAR; ++i) tc::mbar_init(bar(i), (i == B_PA || i == B_PB) ? 4 : 1);
    *abort_flag = 0;
    tc::fence_mbar_init();
  }
  if (warp == 5) {
    tc::tmem_alloc(sbase + SM::SLOT_OFF, kTmemCols);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sgen + SM::SLOT_OFF);
  // S at column 0 (P, as bf16 pairs, in its columns 64..127), O at column 128

  if (warp == 4) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tc::tma_prefetch_desc(&tmQ);
      tc::tma_prefetch_desc(&tmK);
      tc::tma_prefetch_desc(&tmV);
      tc::mbar_expect_tx(bar(B_QF), SM::Q_BYTES);
#pragma unroll
      for (int s = 0; s < NSUB; ++s) tc::tma_load_4d(sQ + s * kSub, &tmQ, bar(B_QF), s * 64, jq, r0, b);
      for (int i = 0; i < nkv; ++i) {
        const int c0 = (kt_lo + i) * kBN;
        // K(i) once S(i-1) has read K(i-1); V(i) once PV(i-1) has read V(i-1)
        if (i > 0 && !tc::mbar_wait(bar(B_KE), (i - 1) & 1, abort_flag, p.status)) break;
        tc::mbar_expect_tx(bar(B_KF), SM::KV_BYTES);
#pragma unroll
        for (int s = 0; s < NSUB; ++s) tc::tma_load_4d(sK + s * kSub, &tmK, bar(B_KF), s * 64, jk, c0, b);
        if (i > 0 && !tc::mbar_wait(bar(B_VE), (i - 1) & 1, abort_flag, p.status)) break;
        tc::mbar_expect_tx(bar(B_VF), SM::KV_BYTES);
#pragma unroll
        for (int s = 0; s < NSUB; ++s) tc::tma_load_4d(sV + s * kSub, &tmV, bar(B_VF), s * 64, jk, c0, b);
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------- MMA issuer
    constexpr uint32_t idS = tc::idesc_bf16_f32(kBM, kBN, 0, 0);
    constexpr uint32_t idO = tc::idesc_bf16_f32(kBM, D, 0, 1);
    auto issue_S = [&]() {
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = (kk >> 2) * kSub + (kk & 3) * 32;
        tc::mma_ss_elect(tmem, tc::smem_desc_sw128(sQ + off, 16, 1024), tc::smem_desc_sw128(sK + off, 16, 1024),
                         idS, kk > 0);
      }
      tc::mma_commit_elect(bar(B_SF));
      tc::mma_commit_elect(bar(B_KE));
    };
    bool ok = nkv > 0 && tc::mbar_wait_warp(bar(B_QF), 0, abort_flag, p.status) &&
              tc::mbar_wait_warp(bar(B_KF), 0, abort_flag, p.status);
    if (ok) {
      tc::tc_fence_after();
      issue_S();
    }
    for (int i = 0; ok && i < nkv; ++i) {
      const int j = kt_lo + i;
      ok = tc::mbar_wait_warp(bar(B_PA), i & 1, abort_flag, p.status) &&
           tc::mbar_wait_warp(bar(B_VF), i & 1, abort_flag, p.status);
      if (!ok) break;
      tc::tc_fence_after();
#pragma unroll
      for (int kk = kBN / 32; kk < kBN / 16; ++kk)
        tc::mma_ts_elect(tmem + 128, tmem + 64 + kk * 8, tc::smem_desc_sw128(sV + kk * 2048, kSub, 1024), idO,
                         (j > kt_lo || kk > kBN / 32) ? 1u : 0u);
      ok = tc::mbar_wait_warp(bar(B_PB), i & 1, abort_flag, p.status);
      if (!ok) break;
      tc::tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < kBN / 32; ++kk)
        tc::mma_ts_elect(tmem + 128, tmem + 64 + kk * 8, tc::smem_desc_sw128(sV + kk * 2048, kSub, 1024), idO,
                         1u);
      tc::mma_commit_elect(bar(B_VE));
      if (j == kt_hi) tc::mma_commit_elect(bar(B_OF));
      if (i + 1 < nkv) {
        ok = tc::mbar_wait_warp(bar(B_KF), (i + 1) & 1, abort_flag, p.status);
        if (!ok) break;
        tc::tc_fence_after();
        issue_S();
      }
    }
  } else {
    const int row = tid;
    const int r = r0 + row;
    const uint32_t tq = static_cast<uint32_t>(warp * 32) << 16;  // this warp's TMEM lanes
    const uint32_t tS = tmem + tq, tO = tS + 128;
    const int hi_r = p.a * r + p.bb;
    const int lo_r = hi_r - p.win;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    int t = 0;
    for (int j = kt_lo; j <= kt_hi; ++j, ++t) {
      if (!tc::mbar_wait(bar(B_SF), t & 1, abort_flag, p.status)) { ok = false; break; }
      tc::tc_fence_after();
      const int c0 = j * kBN;
      const bool full = (c0 + kBN - 1 <= p.a * r0 + p.bb) &&
                        (c0 > p.a * rq_last + p.bb - p.win) && (c0 + kBN <= p.Lk);
      // The row's 128 scores are read from TMEM once and stay in registers
      // (158 registers per thread, under the 168 that two CTAs of 6 warps allow).
      // P goes to columns 64..127 as bf16 pairs (keys 0-63 -> 64..95,
      // keys 64-127 -> 96..127), i.e. only over scores already read.
      auto mask32 = [&](uint32_t* v, int k0) {
        if (!full) {
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int key = c0 + k0 + e;
            if (!(key <= hi_r && key > lo_r && key < p.Lk)) v[e] = __float_as_uint(-INFINITY);
          }
        }
      };
      // P of 32 keys -> 16 TMEM columns. The exponent s*scale*log2(e) - m of a
      // pair of keys is one paired fp32 FMA (fma.rn.f32x2: each half rounds
      // like fmaf), which frees issue slots for the exponentials: 4-6 %
      // faster at the power cap than one fmaf per key.
      auto exp32 = [&](const uint32_t* v, uint32_t col, float m_use) {
        uint32_t pk[16];
        const uint64_t sc2 = pack_f32x2(p.scale_log2, p.scale_log2);
        const uint64_t nm2 = pack_f32x2(-m_use, -m_use);
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          float x0, x1;
          fma_f32x2(v[e], v[e + 1], sc2, nm2, x0, x1);
          const float p0 = fast_exp2(x0);
          const float p1 = fast_exp2(x1);
          l_run += p0 + p1;
          pk[e >> 1] = pack_bf16(p0, p1);
        }
        tc::tmem_st16(tS + col, pk);
      };
      // the values of a tcgen05.ld are only defined after tcgen05.wait::ld:
      // an empty asm on each register keeps every use behind the wait
      auto pin32 = [](uint32_t* v) {
#pragma unroll
        for (int e = 0; e < 32; ++e) asm volatile("" : "+r"(v[e]));
      };
      uint32_t v1[64];
      uint32_t v[64];
      float mx;
      {
        tc::tmem_ld32(tS, v);
        tc::tmem_ld32(tS + 32, v + 32);
        tc::tmem_ld32(tS + 64, v1);
        tc::tmem_ld32(tS + 96, v1 + 32);
        tc::tmem_wait_ld();
        pin32(v); pin32(v + 32); pin32(v1); pin32(v1 + 32);
        mask32(v, 0); mask32(v + 32, 32); mask32(v1, 64); mask32(v1 + 32, 96);
        float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
        for (int e = 0; e < 64; e += 2) {
          m0 = fmaxf(m0, fmaxf(__uint_as_float(v[e]), __uint_as_float(v[e + 1])));
          m1 = fmaxf(m1, fmaxf(__uint_as_float(v1[e]), __uint_as_float(v1[e + 1])));
        }
        mx = fmaxf(m0, m1);
      }
      const float m_tile = mx * p.scale_log2;
      const bool need = m_tile > m_run + kRescaleLog2;
      if (__any_sync(0xffffffffu, need)) {
        const float m_new = fmaxf(m_run, m_tile);
        const float alpha = (m_run == -INFINITY) ? 0.f : fast_exp2(m_run - m_new);
        if (t > 0) {
          // 8 columns at a time: all 128 scores of the row are live here
#pragma unroll 1
          for (int c = 0; c < D / 8; ++c) {
            uint32_t o[8];
            tc::tmem_ld8(tO + c * 8, o);
            tc::tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 8; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            tc::tmem_st8(tO + c * 8, o);
          }
        }
        l_run *= alpha;
        m_run = m_new;
      }
      const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
      exp32(v1, 96, m_use);
      exp32(v1 + 32, 112, m_use);
      tc::tmem_wait_st();
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(bar(B_PA));
      exp32(v, 64, m_use);
      exp32(v + 32, 80, m_use);
      tc::tmem_wait_st();
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(bar(B_PB));
    }
    const bool has_rows = nkv > 0;
    // warp-uniform, every lane taking part (the tcgen05.ld of O below needs
    // the whole warp)
    if (has_rows) ok = tc::mbar_wait_warp(bar(B_OF), 0, abort_flag, p.status) && ok;
    ok = __all_sync(0xffffffffu, ok);
    if (ok && has_rows) {
      tc::tc_fence_after();
      const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
      // O row -> bf16 -> shared memory (the Q tile's space, same swizzled layout)
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tc::tmem_ld32(tO + c * 32, o);
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
        if (in_bounds(li, 1, p.ext_lse, p.status))
          p.lse[li] = (m_run + __log2f(l_run)) * 0.69314718055994530942f;
      }
      tc::fence_async_smem();
    }
    asm volatile("bar.sync 1, 128;\n" ::: "memory");  // the softmax warps only
    if (row == 0 && ok && has_rows && !*abort_flag) {
#pragma unroll
      for (int s = 0; s < NSUB; ++s) tc::tma_store_4d(&tmO, sQ + s * kSub, s * 64, jq, r0, b);
      tc::tma_store_commit_and_wait();
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 5) {
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
  const long long num_qt = (p.Lq + kBM - 1) / kBM;
  const long long blocks = num_qt * p.B * p.Hq * p.groups;
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
