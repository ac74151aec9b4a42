// attn_bwd_tc.cu - Stream-Factorized attention backward on tcgen05 + TMEM + TMA.
//
// Gradients of O = softmax(scale Q K^T over visible keys) V (page "微信WeLM提出
// Hidden Decoding：大模型推理新范式", tahou.com, section "规模化落地的工程优化"):
//   P_ij = exp(scale q_i.k_j - LSE_i), dP = dO V^T, dS = P * (dP - D),
//   dQ = scale dS K,  dK = scale sum_group dS^T Q,  dV = sum_group P^T dO.
//
// One CTA owns 128 keys of one (batch, KV head, stream group) and loops over
// the query heads of its GQA group and the 64-row query tiles that can see its
// keys. Per query tile, on the tensor cores (one issuing thread, fp32 in TMEM):
//   S^T  = K Q^T      (M 128 keys, N 64 queries)   } double-buffered in TMEM
//   dP^T = V dO^T     (M 128 keys, N 64 queries)   }
//   dV  += P^T dO     (M 128 keys, N D; P^T in TMEM) } accumulated in TMEM across
//   dK  += dS^T Q     (M 128 keys, N D; dS^T in TMEM) } the whole group
//   dQ^T = K^T dS^T   (M D, N 64 queries)           into the S^T buffer
// Roles (15 warps):
//   warps 0-7   two warpgroups, one key row per thread, each taking 32 of the
//               64 query columns: P^T = exp2(S^T - LSE), dS^T = P^T (dP^T - D).
//               P^T and dS^T go as bf16 pairs into TMEM, over the warpgroup's
//               own S^T and dP^T columns once they are read (the A operands of
//               dV and dK), and dS^T also into shared memory in the MMA operand
//               layout (the B operand of dQ^T). At the end warpgroup 0 stores
//               dK (scaled) and warpgroup 1 dV through TMA.
//   warps 8-11  one head-dim row per thread: dQ^T from TMEM into an fp32 tile
//               in shared memory, added into the fp32 dQ accumulator by a TMA
//               bulk reduce-add (the TMA unit does the adds, not the SM).
//   warp 12     TMA: K, V once; Q and dO tiles (3 stages) plus the tile's
//               packed LSE and D rows (bulk copies).
//   warp 13     TMEM allocation; issues dV, dK and dQ^T.
//   warp 14     issues S^T and dP^T of the next tile.
// Each issuer warp walks its loop as a whole warp (warp-uniform operands) and
// one elected lane issues. The two groups wait on different barriers (P^T
// written vs. the next stage loaded and its buffer free), so each has its own
// warp; their hand-offs go through the barriers below, not issue order.
// The grid walks key tiles heavy-first, in buckets that keep a problem's
// neighbouring key tiles running together where that helps L2 reuse (below).
// Every mbarrier wait is bounded (HD_ERR_TIMEOUT, then every role leaves).
#include <cuda.h>

#include "hd_common.cuh"
#include "launch.h"
#include "tc_ptx.cuh"

namespace hd {

namespace {

constexpr int kKN = 128;   // keys per CTA
constexpr int kQM = 64;    // query rows per iteration
constexpr int kQS = 3;     // Q / dO stages
constexpr int kThreads = 480;
constexpr int kKB = 8;         // key tiles per grid bucket (INTRA, short windows)
constexpr int kLongKT = 512;   // a problem this many key tiles long is one bucket
constexpr uint32_t kTmemCols = 512;

template <int D>
struct BtSmem {
  static constexpr int NSUB = D / 64;
  static constexpr int KSUB = kKN * 128;    // [128 rows][64 bf16] sub-tile
  static constexpr int QSUB = kQM * 128;    // [64 rows][64 bf16] sub-tile
  static constexpr int K_OFF = 0;
  static constexpr int V_OFF = K_OFF + NSUB * KSUB;
  static constexpr int Q_OFF = V_OFF + NSUB * KSUB;          // kQS stages
  static constexpr int DO_OFF = Q_OFF + kQS * NSUB * QSUB;   // kQS stages
  static constexpr int DS_OFF = DO_OFF + kQS * NSUB * QSUB;  // [128 keys][64 q] bf16
  static constexpr int DQ_OFF = DS_OFF + kKN * 128;          // D/32 boxes of [64 q][32] fp32
  static constexpr int L_OFF = DQ_OFF + (D / 32) * kQM * 32 * 4;  // kQS stages x 64 LSE (log2)
  static constexpr int DL_OFF = L_OFF + kQS * kQM * 4;            // kQS stages x 64 D
  static constexpr int BAR_OFF = DL_OFF + kQS * kQM * 4;
  static constexpr int NBAR = 16;
  static constexpr int SLOT_OFF = BAR_OFF + NBAR * 8;
  static constexpr int ABORT_OFF = SLOT_OFF + 4;
  static constexpr int USED = ABORT_OFF + 4 + 1024;
  static_assert(USED <= 232448, "shared memory");
  // at least 120 KB: one CTA (one 512-column TMEM allocation) per SM
  static constexpr int TOTAL = USED > 120 * 1024 ? USED : 120 * 1024;
};

// barrier indices
enum {
  B_KV = 0,   // K and V loaded
  B_QF = 1,   // [kQS] Q, dO and the packed LSE / D rows of a stage loaded
  B_QE = 4,   // [kQS] stage free (one MMA commit from each issuer)
  B_SF = 7,   // [2] S^T / dP^T ready (MMA commit)
  B_PF = 9,   // P^T / dS^T written (8 warp arrivals)
  B_PE = 10,  // dS^T in shared memory consumed by the MMAs (MMA commit)
  B_DF = 11,  // [2] dQ^T ready (MMA commit)
  B_DE = 13,  // [2] dQ^T read out (4 warp arrivals)
  B_END = 15  // every MMA done (MMA commit)
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_bwd_tc_kernel(const AttnParams p, const __grid_constant__ CUtensorMap tmQ,
                       const __grid_constant__ CUtensorMap tmDO, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDK,
                       const __grid_constant__ CUtensorMap tmDV, const __grid_constant__ CUtensorMap tmDQ) {
  using SM = BtSmem<D>;
  constexpr int NSUB = SM::NSUB;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - smem_u32(smem_raw));
  const uint32_t sK = sbase + SM::K_OFF, sV = sbase + SM::V_OFF, sQ = sbase + SM::Q_OFF,
                 sDO = sbase + SM::DO_OFF, sDS = sbase + SM::DS_OFF, sDQ = sbase + SM::DQ_OFF;
  float* sL = reinterpret_cast<float*>(sgen + SM::L_OFF);
  float* sDl = reinterpret_cast<float*>(sgen + SM::DL_OFF);
  auto bar = [&](int i) { return sbase + SM::BAR_OFF + 8u * i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sgen + SM::ABORT_OFF);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (p.status && *reinterpret_cast<volatile int*>(p.status) == HD_ERR_TIMEOUT) return;

  // ---- problem of this CTA: key tile kt of (b, hk, grp). The grid walks
  // buckets of key tiles, low buckets (which see the most queries) first.
  // Inside a bucket a problem's key tiles are adjacent, so they run at the
  // same time and share their Q, dO and dQ tiles in L2. Buckets of kKB key
  // tiles for INTRA problems (one stream each, many of them) and for windows
  // short against the sequence (key tiles of nearly equal work). A problem of
  // at least kLongKT key tiles is one bucket: the CTAs running at once then
  // hold one problem's key tiles instead of a slice of every problem, and walk
  // its query tiles together (the KV-mirror backward at 131072 keys: 5 %
  // faster than key-tile-major, DRAM traffic 23.5 -> 6.6 GB). Other problems
  // take one key tile per bucket (key-tile-major), which measured best there.
  const int bkg = p.B * p.Hkv * p.groups;
  const int num_kt = (p.Lk + kKN - 1) / kKN;
  const bool bucketed = p.groups > 1 || 4LL * p.win <= p.Lk;
  const int kb = bucketed ? min(kKB, num_kt) : (num_kt >= kLongKT ? num_kt : 1);
  const int bucket = static_cast<int>(blockIdx.x / (bkg * kb));
  const int rem = static_cast<int>(blockIdx.x - static_cast<long long>(bucket) * bkg * kb);
  const int bsize = min(kb, num_kt - bucket * kb);
  const int kt = bucket * kb + rem % bsize;
  int y = rem / bsize;
  const int grp = y % p.groups;
  y /= p.groups;
  const int hk = y % p.Hkv;
  const int b = y / p.Hkv;
  const int g = p.Hq / p.Hkv;
  const bool intra = p.mode == HD_INTRA;
  const int jk = intra ? (p.final_only ? p.n - 1 : grp) * p.Hkv + hk : hk;
  const int c0 = kt * kKN;
  const int c_last = min(c0 + kKN, p.Lk) - 1;
  const int rmin = (c0 - p.bb <= 0) ? 0 : (c0 - p.bb + p.a - 1) / p.a;
  const int rmax = min(p.Lq - 1, (c_last + p.win - 1 - p.bb) / p.a);
  const int qt_lo = rmin / kQM, qt_hi = rmax / kQM;
  const int nqt = rmin <= rmax ? qt_hi - qt_lo + 1 : 0;
  const int total = g * nqt;
  // Query tiles from the last one down, the group's heads inner: the CTAs of
  // one (batch, KV head) then walk the same tiles at the same time, so Q, dO
  // and the dQ accumulator tiles they share stay in L2.
  auto iter_head = [&](int it) { return hk * g + it % g; };
  auto iter_row0 = [&](int it) { return (qt_hi - it / g) * kQM; };
  auto jq_of = [&](int h) { return (intra && !p.final_only) ? grp * p.Hq + h : h; };

  if (tid == 0) {
    for (int i = 0; i < SM::NBAR; ++i) {
      uint32_t cnt = 1;
      if (i == B_DE || i == B_DE + 1) cnt = 4;
      if (i >= B_QE && i < B_QE + kQS) cnt = 2;
      if (i == B_PF) cnt = 8;
      tc::mbar_init(bar(i), cnt);
    }
    *abort_flag = 0;
    tc::fence_mbar_init();
  }
  if (warp == 13) {
    tc::tmem_alloc(sbase + SM::SLOT_OFF, kTmemCols);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sgen + SM::SLOT_OFF);
  // TMEM columns: buffer x in {0,1}: S^T at 128x, dP^T at 128x + 64 (dQ^T reuses S^T);
  // dK at 256, dV at 256 + D.
  const uint32_t tdK = tmem + 256, tdV = tmem + 256 + D;

  if (warp == 12) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tc::tma_prefetch_desc(&tmQ);
      tc::tma_prefetch_desc(&tmDO);
      tc::mbar_expect_tx(bar(B_KV), 2 * NSUB * SM::KSUB);
#pragma unroll
      for (int s = 0; s < NSUB; ++s) {
        tc::tma_load_4d(sK + s * SM::KSUB, &tmK, bar(B_KV), s * 64, jk, c0, b);
        tc::tma_load_4d(sV + s * SM::KSUB, &tmV, bar(B_KV), s * 64, jk, c0, b);
      }
    }
    for (int it = 0; lane == 0 && it < total; ++it) {
      const int st = it % kQS;
      if (!tc::mbar_wait(bar(B_QE + st), ((it / kQS) & 1) ^ 1, abort_flag, p.status)) break;
      const int h = iter_head(it), rq0 = iter_row0(it), jq = jq_of(h);
      if (lane == 0) {
        const long long pk = ((static_cast<long long>(b) * p.Hq + h) * p.groups + grp) * p.lq_pad + rq0;
        if (!in_bounds(pk, kQM, p.ext_packed, p.status)) {  // checked build only
          *abort_flag = 1;
          break;
        }
        tc::mbar_expect_tx(bar(B_QF + st), 2 * NSUB * SM::QSUB + 2 * kQM * 4);
#pragma unroll
        for (int s = 0; s < NSUB; ++s) {
          tc::tma_load_4d(sQ + (st * NSUB + s) * SM::QSUB, &tmQ, bar(B_QF + st), s * 64, jq, rq0, b);
          tc::tma_load_4d(sDO + (st * NSUB + s) * SM::QSUB, &tmDO, bar(B_QF + st), s * 64, jq, rq0, b);
        }
        tc::bulk_load(sbase + SM::L_OFF + st * kQM * 4, p.lse2p + pk, kQM * 4, bar(B_QF + st));
        tc::bulk_load(sbase + SM::DL_OFF + st * kQM * 4, p.deltap + pk, kQM * 4, bar(B_QF + st));
      }
    }
  } else if (warp == 13 || warp == 14) {
    // ------------------------------------------------------------ MMA issuers
    if (total > 0) {  // the whole warp walks the issue loop; one elected lane issues
      constexpr uint32_t idSP = tc::idesc_bf16_f32(128, kQM, 0, 0);  // S^T, dP^T
      constexpr uint32_t idKV = tc::idesc_bf16_f32(128, D, 0, 1);    // dV, dK
      constexpr uint32_t idDQ = tc::idesc_bf16_f32(128, kQM, 1, 1);  // dQ^T
      // rows 64..127 of K^T for D = 64 read the V tile and are ignored
      constexpr uint32_t kt_lbo = (D == 64) ? (SM::V_OFF - SM::K_OFF) : SM::KSUB;
      // Base descriptors, built once; a k-step only adds its byte offset / 16
      // to the start-address field.
      const uint64_t dK = tc::smem_desc_sw128(sK, 16, 1024), dV = tc::smem_desc_sw128(sV, 16, 1024);
      const uint64_t dQk = tc::smem_desc_sw128(sQ, 16, 1024), dOk = tc::smem_desc_sw128(sDO, 16, 1024);
      const uint64_t dQm = tc::smem_desc_sw128(sQ, SM::QSUB, 1024), dOm = tc::smem_desc_sw128(sDO, SM::QSUB, 1024);
      const uint64_t dS = tc::smem_desc_sw128(sDS, 16, 1024);
      const uint64_t dSm = tc::smem_desc_sw128(sDS, SM::QSUB, 1024);
      const uint64_t dKt = tc::smem_desc_sw128(sK, kt_lbo, 1024);
      auto add = [](uint64_t d, uint32_t bytes) { return d + (bytes >> 4); };
      bool ok = tc::mbar_wait_warp(bar(B_KV), 0, abort_flag, p.status);
      if (warp == 14) {
        // S^T, dP^T of tile it into TMEM buffer it & 1, once the stage is
        // loaded and dQ^T of tile it-2 (same buffer) has been read out
        for (int it = 0; ok && it < total; ++it) {
          const int x = it & 1, st = it % kQS;
          ok = tc::mbar_wait_warp(bar(B_QF + st), (it / kQS) & 1, abort_flag, p.status);
          if (ok && it >= 2) ok = tc::mbar_wait_warp(bar(B_DE + x), ((it >> 1) - 1) & 1, abort_flag, p.status);
          if (!ok) break;
          tc::tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t ko = (kk >> 2) * SM::KSUB + (kk & 3) * 32;
            const uint32_t qo = (st * NSUB + (kk >> 2)) * SM::QSUB + (kk & 3) * 32;
            tc::mma_ss_elect(tmem + 128 * x, add(dK, ko), add(dQk, qo), idSP, kk > 0);
            tc::mma_ss_elect(tmem + 128 * x + 64, add(dV, ko), add(dOk, qo), idSP, kk > 0);
          }
          tc::mma_commit_elect(bar(B_SF + x));
          tc::mma_commit_elect(bar(B_QE + st));
        }
      } else {
        // dV, dK, dQ^T of tile it once P^T / dS^T are written
        for (int it = 0; ok && it < total; ++it) {
          const int x = it & 1, st = it % kQS;
          ok = tc::mbar_wait_warp(bar(B_QF + st), (it / kQS) & 1, abort_flag, p.status) &&
               tc::mbar_wait_warp(bar(B_PF), it & 1, abort_flag, p.status);
          if (!ok) break;
          tc::tc_fence_after();
          const uint32_t acc = it > 0 ? 1u : 0u;
#pragma unroll
          for (int kk = 0; kk < kQM / 16; ++kk) {  // reduce over the 64 queries
            // P^T of queries 16kk..16kk+15: warpgroup kk/2 wrote its 32
            // queries at S^T columns 32*(kk/2)..+15 of buffer x, two per column
            // (dS^T likewise at the dP^T columns, 64 further on)
            const uint32_t ap = tmem + 128 * x + (kk >> 1) * 32 + (kk & 1) * 8;
            const uint64_t bo = add(dOm, st * NSUB * SM::QSUB + kk * 2048);
            const uint64_t bq = add(dQm, st * NSUB * SM::QSUB + kk * 2048);
            tc::mma_ts_elect(tdV, ap, bo, idKV, (acc | kk) ? 1u : 0u);
            tc::mma_ts_elect(tdK, ap + 64, bq, idKV, (acc | kk) ? 1u : 0u);
          }
#pragma unroll
          for (int kk = 0; kk < kKN / 16; ++kk) {  // reduce over the 128 keys
            const uint64_t ak = add(dKt, kk * 2048);
            const uint64_t bs = add(dSm, kk * 2048);
            tc::mma_ss_elect(tmem + 128 * x, ak, bs, idDQ, kk > 0 ? 1u : 0u);
          }
          tc::mma_commit_elect(bar(B_DF + x));
          tc::mma_commit_elect(bar(B_QE + st));
          tc::mma_commit_elect(bar(B_PE));
        }
        // every S^T / dP^T MMA finished before the last P^T was written, so this
        // covers both issuers
        tc::mma_commit_elect(bar(B_END));
      }
    }
  } else if (warp < 8) {
    // ------------------------- P^T, dS^T: one key per thread, warpgroup sw takes
    // query columns 32*sw .. 32*sw+31
    const int sw = warp >> 2;
    const int row = tid & 127;
    const int c = c0 + row;
    const uint32_t tq = static_cast<uint32_t>((warp & 3) * 32) << 16;
    // The query rows this thread's key is visible to, r_lo .. r_hi (empty when
    // r_lo > r_hi), from the visibility rule c <= a*r + bb, c > a*r + bb - win,
    // r < Lq, c < Lk; fixed for the whole CTA. c - bb + win - 1 >= 0 always,
    // since win >= a (a window spans at least one token's n positions).
    int r_lo = 1, r_hi = 0;
    if (c < p.Lk) {
      r_lo = (c - p.bb <= 0) ? 0 : (c - p.bb + p.a - 1) / p.a;
      const long long num = static_cast<long long>(c) - p.bb + p.win - 1;
      r_hi = static_cast<int>(min(static_cast<long long>(p.Lq - 1), num / p.a));
    }
    bool ok = true;
    for (int it = 0; it < total; ++it) {
      const int x = it & 1, st = it % kQS;
      const int rq0 = iter_row0(it);
      if (!tc::mbar_wait(bar(B_SF + x), (it >> 1) & 1, abort_flag, p.status)) { ok = false; break; }
      tc::tc_fence_after();
      const bool full = (c0 + kKN - 1 <= p.a * rq0 + p.bb) &&
                        (c0 > p.a * (rq0 + kQM - 1) + p.bb - p.win) && (c0 + kKN <= p.Lk) &&
                        (rq0 + kQM <= p.Lq);
      uint32_t pp[16], dd[16];  // bf16 pairs of P^T and dS^T for this warpgroup's 32 queries
      {
        uint32_t sr[32], dr[32];
        tc::tmem_ld32(tmem + tq + 128 * x + sw * 32, sr);
        tc::tmem_ld32(tmem + tq + 128 * x + 64 + sw * 32, dr);
        tc::tmem_wait_ld();
        // The mask is a separate pass (score -> -inf, so P and dS become 0):
        // a test inside the arithmetic loop below would serialise it.
        if (!full) {
          const int elo = r_lo - (rq0 + sw * 32), ehi = r_hi - (rq0 + sw * 32);
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (e < elo || e > ehi) sr[e] = __float_as_uint(-INFINITY);
        }
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
          const float4 l4 = *reinterpret_cast<const float4*>(sL + st * kQM + sw * 32 + j);
          const float4 d4 = *reinterpret_cast<const float4*>(sDl + st * kQM + sw * 32 + j);
          const float lv[4] = {l4.x, l4.y, l4.z, l4.w};
          const float dv4[4] = {d4.x, d4.y, d4.z, d4.w};
          float pj[4], dj[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float pv = fast_exp2(fmaf(__uint_as_float(sr[j + e]), p.scale_log2, -lv[e]));
            pj[e] = pv;
            dj[e] = pv * (__uint_as_float(dr[j + e]) - dv4[e]);
          }
          pp[j / 2] = pack_bf16(pj[0], pj[1]);
          pp[j / 2 + 1] = pack_bf16(pj[2], pj[3]);
          dd[j / 2] = pack_bf16(dj[0], dj[1]);
          dd[j / 2 + 1] = pack_bf16(dj[2], dj[3]);
        }
      }
      // P^T and dS^T into TMEM over this warpgroup's own S^T and dP^T columns,
      // read above. The S^T columns next take this tile's dQ^T, which the MMAs
      // write only after dV has read P^T: MMAs from one thread execute in
      // order. (Shared-memory operands cost bandwidth the MMAs need: each of
      // these moves was 1-2 % faster.)
      tc::tmem_st16(tmem + tq + 128 * x + sw * 32, pp);
      tc::tmem_st16(tmem + tq + 128 * x + 64 + sw * 32, dd);
      // the MMAs of the previous tile have finished reading dS^T
      if (it > 0) {
        if (!tc::mbar_wait(bar(B_PE), (it - 1) & 1, abort_flag, p.status)) { ok = false; break; }
      }
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int ch = sw * 4 + k;
        const uint32_t off = row * 128 + ((ch ^ (row & 7)) << 4);
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};\n" ::"r"(sDS + off), "r"(dd[4 * k]),
                     "r"(dd[4 * k + 1]), "r"(dd[4 * k + 2]), "r"(dd[4 * k + 3])
                     : "memory");
      }
      tc::tmem_wait_st();
      tc::fence_async_smem();
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(bar(B_PF));
    }
    // ---- warpgroup 0: dK (scaled), warpgroup 1: dV; TMEM -> bf16 -> shared
    // memory (the Q / dO stages) -> TMA store
    // warp-uniform (the tcgen05.ld below needs the whole warp)
    if (total > 0) ok = tc::mbar_wait_warp(bar(B_END), 0, abort_flag, p.status) && ok;
    ok = __all_sync(0xffffffffu, ok && !*abort_flag);
    const uint32_t src = sw == 0 ? tdK : tdV;
    const uint32_t dst = sw == 0 ? sQ : sDO;  // kQS x NSUB x [64][64] >= NSUB x [128][64]
    const float sc = sw == 0 ? p.scale : 1.f;
    if (ok) {
      tc::tc_fence_after();
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t v[32];
        if (total > 0) {
          tc::tmem_ld32(src + tq + cc * 32, v);
          tc::tmem_wait_ld();
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = 0u;
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int d8 = cc * 4 + k;
          const float* f = reinterpret_cast<const float*>(v + 8 * k);
          const uint32_t addr = dst + (d8 >> 3) * SM::KSUB + row * 128 + (((d8 & 7) ^ (row & 7)) << 4);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};\n" ::"r"(addr),
                       "r"(pack_bf16(f[0] * sc, f[1] * sc)), "r"(pack_bf16(f[2] * sc, f[3] * sc)),
                       "r"(pack_bf16(f[4] * sc, f[5] * sc)), "r"(pack_bf16(f[6] * sc, f[7] * sc))
                       : "memory");
        }
      }
      tc::fence_async_smem();
    }
    if (sw == 0) asm volatile("bar.sync 1, 128;\n" ::: "memory");
    else asm volatile("bar.sync 2, 128;\n" ::: "memory");
    if (row == 0 && ok && !*abort_flag) {
#pragma unroll
      for (int s = 0; s < NSUB; ++s) tc::tma_store_4d(sw == 0 ? &tmDK : &tmDV, dst + s * SM::KSUB, s * 64, jk, c0, b);
      tc::tma_store_commit_and_wait();
    }
  } else if (warp < 12) {
    // ------------------- dQ^T read-out (one head-dim row per thread), added into
    // the fp32 accumulator with coalesced reductions (32 consecutive d per warp)
    const int d = tid - 256;
    const uint32_t tq = static_cast<uint32_t>((warp & 3) * 32) << 16;
    for (int it = 0; it < total; ++it) {
      const int x = it & 1;
      if (!tc::mbar_wait(bar(B_DF + x), (it >> 1) & 1, abort_flag, p.status)) break;
      tc::tc_fence_after();
      uint32_t v0[32], v1[32];
      tc::tmem_ld32(tmem + tq + 128 * x, v0);
      tc::tmem_ld32(tmem + tq + 128 * x + 32, v1);
      tc::tmem_wait_ld();
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(bar(B_DE + x));
      // the previous reduce-add has finished reading the staging tile
      if (d == 0) asm volatile("cp.async.bulk.wait_group.read 0;\n" ::: "memory");
      asm volatile("bar.sync 3, 128;\n" ::: "memory");
      if (d < D) {
        float* stg = reinterpret_cast<float*>(sgen + SM::DQ_OFF) + (d >> 5) * (kQM * 32) + (d & 31);
#pragma unroll
        for (int q = 0; q < 32; ++q) stg[q * 32] = __uint_as_float(v0[q]);
#pragma unroll
        for (int q = 0; q < 32; ++q) stg[(q + 32) * 32] = __uint_as_float(v1[q]);
      }
      tc::fence_async_smem();
      asm volatile("bar.sync 3, 128;\n" ::: "memory");
      if (d == 0) {
        const int h = iter_head(it), rq0 = iter_row0(it), jq = jq_of(h);
#pragma unroll
        for (int bx = 0; bx < D / 32; ++bx)
          asm volatile(
              "cp.reduce.async.bulk.tensor.4d.global.shared::cta.add.tile.bulk_group"
              " [%0, {%2, %3, %4, %5}], [%1];\n" ::"l"(reinterpret_cast<uint64_t>(&tmDQ)),
              "r"(sDQ + bx * kQM * 32 * 4), "r"(bx * 32), "r"(jq), "r"(rq0), "r"(b)
              : "memory");
        asm volatile("cp.async.bulk.commit_group;\n" ::: "memory");
      }
    }
    if (d == 0) asm volatile("cp.async.bulk.wait_group 0;\n" ::: "memory");
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 13) {
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

// (d, j, row, batch) view; strides in elements; box (box_d, 1, box_rows, 1).
bool make_map(CUtensorMap* map, const void* base, bool fp32, int D, long long J, long long R,
              long long B, long long stride_j, long long stride_r, long long stride_b, int box_d,
              int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const int es = fp32 ? 4 : 2;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(J),
                              static_cast<cuuint64_t>(R), static_cast<cuuint64_t>(B)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(stride_j * es),
                                 static_cast<cuuint64_t>(stride_r * es),
                                 static_cast<cuuint64_t>(stride_b * es)};
  const cuuint32_t box[4] = {static_cast<cuuint32_t>(box_d), 1, static_cast<cuuint32_t>(box_rows), 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(map, fp32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4,
            const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            fp32 ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
cudaError_t launch_bwd_tc_d(const AttnParams& p, cudaStream_t stream) {
  const long long S = p.S, L = p.L, n = p.n, Hq = p.Hq, Hkv = p.Hkv, B = p.B;
  CUtensorMap mq, mdo, mk, mv, mdk, mdv, mdq;
  const bool intra = p.mode == HD_INTRA;
  long long Jq, Rq, sjq, srq, sbq;
  if (intra && !p.final_only) {
    Jq = n * Hq; Rq = L; sjq = D; srq = n * Hq * D; sbq = S * Hq * D;
  } else {
    Rq = p.final_only ? L : S; Jq = Hq; sjq = D; srq = Hq * D; sbq = Rq * Hq * D;
  }
  long long Jk, Rk, srk, sbk;
  if (intra) {
    Jk = n * Hkv; Rk = L; srk = n * Hkv * D; sbk = S * Hkv * D;
  } else {
    Jk = Hkv; Rk = S; srk = Hkv * D; sbk = S * Hkv * D;
  }
  bool ok = make_map(&mq, p.q, false, D, Jq, Rq, B, sjq, srq, sbq, 64, kQM) &&
            make_map(&mdo, p.dout, false, D, Jq, Rq, B, sjq, srq, sbq, 64, kQM) &&
            make_map(&mdq, p.dq_acc, true, D, Jq, Rq, B, sjq, srq, sbq, 32, kQM) &&
            make_map(&mk, p.k, false, D, Jk, Rk, B, D, srk, sbk, 64, kKN) &&
            make_map(&mv, p.v, false, D, Jk, Rk, B, D, srk, sbk, 64, kKN) &&
            make_map(&mdk, p.dk, false, D, Jk, Rk, B, D, srk, sbk, 64, kKN) &&
            make_map(&mdv, p.dv, false, D, Jk, Rk, B, D, srk, sbk, 64, kKN);
  if (!ok) return cudaErrorInvalidValue;
  const int smem = BtSmem<D>::TOTAL;
  cudaError_t e = cudaFuncSetAttribute(attn_bwd_tc_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const long long blocks = static_cast<long long>((p.Lk + kKN - 1) / kKN) * p.B * p.Hkv * p.groups;
  attn_bwd_tc_kernel<D><<<static_cast<unsigned>(blocks), kThreads, smem, stream>>>(p, mq, mdo, mk, mv,
                                                                                   mdk, mdv, mdq);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_bwd_tc_main(const AttnParams& p, cudaStream_t stream) {
  if (p.D == 64) return launch_bwd_tc_d<64>(p, stream);
  if (p.D == 128) return launch_bwd_tc_d<128>(p, stream);
  return cudaErrorInvalidValue;
}

}  // namespace hd
