// decode.cu - one multi-stream decode step against the interleaved KV cache.
//
// Page "微信WeLM提出Hidden Decoding：大模型推理新范式" (tahou.com): section
// "实验效果与成本分析" - the n streams of the new token are computed in one
// parallel step (not one after another), and decode is bandwidth-bound at small
// batch; section "中间流的作用验证" - every stream keeps its own KV state.
//
// Query s of sequence b sits at p = T*n + s (T = seqlen[b]-1) and reads cache
// positions c with c <= p, plus c % n == s (INTRA) or p - c < n*W (CROSS_WINDOW).
// Final-stream-only decode (section "规模化落地的工程优化", KV-mirror: only the
// last stream passes through the mirror layers) runs the query s = n-1 alone;
// under INTRA it then reads only the final stream's cache rows (every n-th row),
// for which every loaded key is visible.
//
// Split-K: each CTA owns (batch, KV head, 16-row tile of the n*group query
// rows, key chunk). K/V blocks of 64 positions stream once through a 3-stage
// cp.async ring; each warp takes 16 of the 64 keys and keeps its own online
// softmax state, so S = Q K^T and O += P V run as m16n8k16 MMAs with the query
// rows as M. Warps are merged in shared memory and the CTA writes one partial
// (max, sum, unnormalised O) per row; decode_combine merges the chunks.
#include "hd_common.cuh"
#include "launch.h"

namespace hd {

namespace {

constexpr int kDecWarps = 4;
constexpr int kDecThreads = kDecWarps * 32;
constexpr int kDecBlk = 64;  // keys per stage
constexpr int kDecStages = 3;
constexpr float kLn2 = 0.69314718055994530942f;

template <int D>
struct DecSmem {
  static constexpr int RC = D / 8;
  static constexpr int Q_BYTES = 16 * D * 2;
  static constexpr int STAGE = kDecBlk * D * 2 * 2;  // K and V
  static constexpr int TOTAL = Q_BYTES + kDecStages * STAGE;
  static_assert(kDecWarps * 16 * (D + 2) * 4 <= kDecStages * STAGE, "merge buffer");
};

__device__ __forceinline__ bool seq_ok(int T1, int Tcap) { return T1 >= 1 && T1 <= Tcap; }

template <int D>
__global__ void __launch_bounds__(kDecThreads, 2) decode_split_kernel(const DecodeParams p) {
  using SM = DecSmem<D>;
  constexpr int RC = SM::RC;
  constexpr int NDT = D / 8;
  extern __shared__ __align__(128) uint8_t smem[];
  const uint32_t sQ = smem_u32(smem);
  const uint32_t sStage = sQ + SM::Q_BYTES;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  long long idx = blockIdx.x;
  const int mt = static_cast<int>(idx % p.mt);
  idx /= p.mt;
  const int split = static_cast<int>(idx % p.splits);
  idx /= p.splits;
  const int hk = static_cast<int>(idx % p.Hkv);
  const int b = static_cast<int>(idx / p.Hkv);
  const int g = p.Hq / p.Hkv;
  const int rows_pad = p.mt * 16;

  const int T1 = p.seqlen[b];
  const bool ok = seq_ok(T1, p.Tcap);
  if (!ok && tid == 0 && mt == 0 && split == 0 && hk == 0) record_status(p.status, HD_ERR_DEVICE_INDEX);
  const int T = ok ? T1 - 1 : 0;
  // key-space range: [kbeg, kend); with kstride 1 key index = cache position
  const int kend = ok ? T1 * p.kpt : 0;
  const int kbeg = (p.mode == HD_CROSS_WINDOW) ? max(0, T * p.n + p.s0 - p.win + 1) : 0;
  const int cs = kbeg + split * p.chunk;
  const int ce = min(kend, cs + p.chunk);
  const long long part_row0 = (static_cast<long long>(b) * p.Hkv + hk) * rows_pad + mt * 16;

  if (cs >= ce) {  // nothing to read in this chunk
    if (tid < 16 && in_bounds((part_row0 + tid) * p.splits + split, 1, p.ext_part, p.status)) {
      float* ml = p.part_ml + ((part_row0 + tid) * p.splits + split) * 2;
      ml[0] = -INFINITY;
      ml[1] = 0.f;
    }
    return;
  }

  // ---- Q rows of this tile: row i = s*g + j -> q[b, s, hk*g + j, :] (s local to the nq streams)
  for (int i = tid; i < 16 * RC; i += kDecThreads) {
    const int lr = i / RC, ch = i % RC, row = mt * 16 + lr;
    const bool valid = row < p.rows;
    const int s = valid ? row / g : 0, j = valid ? row % g : 0;
    const long long qi = ((static_cast<long long>(b) * p.nq + s) * p.Hq + hk * g + j) * D + ch * 8;
    const bool inb = in_bounds(qi, 8, p.ext_q, p.status);
    cp_async16(sQ + swz(lr, ch, RC), p.q + (inb ? qi : 0), (valid && inb) ? 16 : 0);
  }
  const long long kv_rs = static_cast<long long>(p.Hkv) * D;
  const __nv_bfloat16* kg = p.kc + (static_cast<long long>(b) * p.Tcap * p.n * p.Hkv + hk) * D;
  const __nv_bfloat16* vg = p.vc + (static_cast<long long>(b) * p.Tcap * p.n * p.Hkv + hk) * D;
  const int nblk = (ce - cs + kDecBlk - 1) / kDecBlk;
  auto load_blk = [&](int bi, int st) {
    const int base = cs + bi * kDecBlk;
    const uint32_t dk = sStage + st * SM::STAGE, dv = dk + SM::STAGE / 2;
    for (int i = tid; i < kDecBlk * RC; i += kDecThreads) {
      const int row = i / RC, ch = i % RC, c = base + row;
      const long long pos = p.kres + static_cast<long long>(min(c, ce - 1)) * p.kstride;
      const long long off = pos * kv_rs + ch * 8;
      const bool inb = in_bounds((kg - p.kc) + off, 8, p.ext_cache, p.status);
      const int nb = (c < ce && inb) ? 16 : 0;
      cp_async16(dk + swz(row, ch, RC), inb ? kg + off : p.kc, nb);
      cp_async16(dv + swz(row, ch, RC), inb ? vg + off : p.vc, nb);
    }
  };
  load_blk(0, 0);
  cp_async_commit();
  if (nblk > 1) load_blk(1, 1);
  cp_async_commit();
  cp_async_wait<1>();
  __syncthreads();
  uint32_t qf[D / 16][4];
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk)
    ldsm_x4(sQ + swz(lane & 15, kk * 2 + (lane >> 4), RC), qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3]);

  // per-thread rows lane/4 and lane/4 + 8 of the tile
  int prow[2], srow[2];
  bool rvalid[2];
#pragma unroll
  for (int hr = 0; hr < 2; ++hr) {
    const int row = mt * 16 + (lane >> 2) + hr * 8;
    rvalid[hr] = row < p.rows;
    srow[hr] = p.s0 + (rvalid[hr] ? row / g : 0);
    // the query's own key index: its position, or (final stream alone) its token
    prow[hr] = (p.kstride == 1) ? T * p.n + srow[hr] : T;
  }
  // INTRA: key c is visible iff c % n == s. Blocks start at multiples of 64,
  // so c % n = (block base % n + offset % n) mod n: the offsets' residues are
  // fixed per thread, the base's residue is one modulo per block.
  int om[2][2];
#pragma unroll
  for (int j = 0; j < 2; ++j)
#pragma unroll
    for (int e = 0; e < 2; ++e) om[j][e] = (warp * 16 + j * 8 + (lane & 3) * 2 + e) % p.n;
  float o[NDT][4];
#pragma unroll
  for (int j = 0; j < NDT; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};

  for (int bi = 0; bi < nblk; ++bi) {
    const int st = bi % kDecStages;
    if (bi + 2 < nblk) load_blk(bi + 2, (bi + 2) % kDecStages);
    cp_async_commit();
    cp_async_wait<2>();
    __syncthreads();
    const uint32_t kb = sStage + st * SM::STAGE, vb = kb + SM::STAGE / 2;
    float s[2][4];
#pragma unroll
    for (int j = 0; j < 2; ++j) s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      uint32_t b0, b1, b2, b3;
      ldsm_x4(kb + swz(warp * 16 + (lane & 7) + ((lane >> 4) << 3), kk * 2 + ((lane >> 3) & 1), RC),
              b0, b1, b2, b3);
      mma_bf16_16816(s[0], qf[kk], b0, b1);
      mma_bf16_16816(s[1], qf[kk], b2, b3);
    }
    const int cbase = cs + bi * kDecBlk + warp * 16;
    const int bres = (p.mode == HD_INTRA) ? (cs + bi * kDecBlk) % p.n : 0;
#pragma unroll
    for (int j = 0; j < 2; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int hr = e >> 1;
        const int c = cbase + j * 8 + (lane & 3) * 2 + (e & 1);
        bool vis = rvalid[hr] && c < ce && c <= prow[hr];
        if (p.mode == HD_INTRA) {
          int res = bres + om[j][e & 1];
          res -= (res >= p.n) ? p.n : 0;
          vis = vis && (res == srow[hr]);
        }
        if (p.mode == HD_CROSS_WINDOW) vis = vis && (prow[hr] - c < p.win);
        if (!vis) s[j][e] = -INFINITY;
      }
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      float mx = fmaxf(fmaxf(s[0][2 * hr], s[0][2 * hr + 1]), fmaxf(s[1][2 * hr], s[1][2 * hr + 1]));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const float m_new = fmaxf(m_run[hr], mx * p.scale_log2);
      const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
      const float alpha = fast_exp2(m_run[hr] - m_use);
      m_run[hr] = m_new;
      float rs = 0.f;
#pragma unroll
      for (int j = 0; j < 2; ++j) {
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
    uint32_t a[4];
    a[0] = pack_bf16(s[0][0], s[0][1]);
    a[1] = pack_bf16(s[0][2], s[0][3]);
    a[2] = pack_bf16(s[1][0], s[1][1]);
    a[3] = pack_bf16(s[1][2], s[1][3]);
#pragma unroll
    for (int dp = 0; dp < D / 16; ++dp) {
      uint32_t b0, b1, b2, b3;
      ldsm_x4_t(vb + swz(warp * 16 + (lane & 7) + (((lane >> 3) & 1) << 3), dp * 2 + (lane >> 4), RC),
                b0, b1, b2, b3);
      mma_bf16_16816(o[2 * dp], a, b0, b1);
      mma_bf16_16816(o[2 * dp + 1], a, b2, b3);
    }
    __syncthreads();
  }
  cp_async_wait<0>();
  __syncthreads();

  // ---- merge the 4 warps' states in shared memory: per warp [16][D+2] floats
  float* mbuf = reinterpret_cast<float*>(smem + SM::Q_BYTES);
  constexpr int RS = D + 2;
#pragma unroll
  for (int hr = 0; hr < 2; ++hr) {
    float l = l_run[hr];
    l += __shfl_xor_sync(0xffffffffu, l, 1);
    l += __shfl_xor_sync(0xffffffffu, l, 2);
    const int lr = (lane >> 2) + hr * 8;
    float* rowp = mbuf + (warp * 16 + lr) * RS;
    if ((lane & 3) == 0) {
      rowp[D] = m_run[hr];
      rowp[D + 1] = l;
    }
#pragma unroll
    for (int j = 0; j < NDT; ++j) {
      const int col = j * 8 + (lane & 3) * 2;
      rowp[col] = o[j][2 * hr];
      rowp[col + 1] = o[j][2 * hr + 1];
    }
  }
  __syncthreads();
  for (int i = tid; i < 16 * D; i += kDecThreads) {
    const int lr = i / D, col = i % D;
    float mw[kDecWarps], mx = -INFINITY;
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) {
      mw[w] = mbuf[(w * 16 + lr) * RS + D];
      mx = fmaxf(mx, mw[w]);
    }
    const float mu = (mx == -INFINITY) ? 0.f : mx;
    float acc = 0.f, lt = 0.f;
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) {
      const float f = fast_exp2(mw[w] - mu);
      acc += f * mbuf[(w * 16 + lr) * RS + col];
      lt += f * mbuf[(w * 16 + lr) * RS + D + 1];
    }
    const long long prow_i = (part_row0 + lr) * p.splits + split;
    if (!in_bounds(prow_i, 1, p.ext_part, p.status)) continue;
    p.part_o[prow_i * D + col] = acc;
    if (col == 0) {
      p.part_ml[prow_i * 2] = mx;
      p.part_ml[prow_i * 2 + 1] = lt;
    }
  }
}

template <int D>
__global__ void decode_combine_kernel(const DecodeParams p) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long gi = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + warp;
  const long long total = static_cast<long long>(p.B) * p.Hkv * p.rows;
  if (gi >= total) return;
  const int row = static_cast<int>(gi % p.rows);
  const int hk = static_cast<int>((gi / p.rows) % p.Hkv);
  const int b = static_cast<int>(gi / (static_cast<long long>(p.rows) * p.Hkv));
  const int g = p.Hq / p.Hkv;
  const int s = row / g, h = hk * g + row % g;  // s local to the nq query streams
  const long long prow = (static_cast<long long>(b) * p.Hkv + hk) * (p.mt * 16) + row;
  const long long oi = ((static_cast<long long>(b) * p.nq + s) * p.Hq + h) * D;
  const long long li = (static_cast<long long>(b) * p.Hq + h) * p.nq + s;
  if (!in_bounds(prow * p.splits, p.splits, p.ext_part, p.status) || !in_bounds(oi, D, p.ext_q, p.status) ||
      !in_bounds(li, 1, p.ext_lse, p.status))
    return;
  const bool ok = seq_ok(p.seqlen[b], p.Tcap);

  float mx = -INFINITY;
  for (int j = lane; j < p.splits; j += 32) mx = fmaxf(mx, p.part_ml[(prow * p.splits + j) * 2]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  const float mu = (mx == -INFINITY) ? 0.f : mx;
  constexpr int PER = D / 32;
  float acc[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) acc[i] = 0.f;
  float lt = 0.f;
  for (int j = 0; j < p.splits; ++j) {
    const float* ml = p.part_ml + (prow * p.splits + j) * 2;
    // a chunk past the end of the sequence wrote only (max, sum) = (-inf, 0);
    // its partial O was never written, so it must not be read
    if (!(ml[1] > 0.f)) continue;
    const float f = fast_exp2(ml[0] - mu);
    lt += f * ml[1];
    const float* po = p.part_o + (prow * p.splits + j) * D;
#pragma unroll
    for (int i = 0; i < PER; ++i) acc[i] += f * po[lane + 32 * i];
  }
  const float inv = (ok && lt > 0.f) ? 1.f / lt : 0.f;
  __nv_bfloat16* out = p.o + oi;
#pragma unroll
  for (int i = 0; i < PER; ++i) out[lane + 32 * i] = __float2bfloat16_rn(acc[i] * inv);
  if (lane == 0) p.lse[li] = (ok && lt > 0.f) ? (mx + __log2f(lt)) * kLn2 : -INFINITY;
}

template <int D>
cudaError_t launch_decode_d(const DecodeParams& p, cudaStream_t stream) {
  const int smem = DecSmem<D>::TOTAL;
  cudaError_t e = cudaFuncSetAttribute(decode_split_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const long long blocks = static_cast<long long>(p.B) * p.Hkv * p.splits * p.mt;
  decode_split_kernel<D><<<static_cast<unsigned>(blocks), kDecThreads, smem, stream>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const long long rows = static_cast<long long>(p.B) * p.Hkv * p.rows;
  decode_combine_kernel<D><<<static_cast<unsigned>((rows + 7) / 8), 256, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

void decode_split_plan(int B, int rows, long long keys, int Hkv, int sms, int* mt, int* splits,
                       int* chunk) {
  const int m = (rows + 15) / 16;
  const long long units = static_cast<long long>(B) * Hkv * m;
  const long long target = static_cast<long long>(sms) * 2 * 4;  // 4 waves of 2 resident CTAs per SM
  long long sp = (target + units - 1) / units;
  // at least 8 blocks (512 keys) per split, so that short caches are not cut
  // into many tiny chunks that the combine step then has to walk
  const long long max_sp = (keys + 8 * kDecBlk - 1) / (8 * kDecBlk);
  if (sp > max_sp) sp = max_sp;
  if (sp < 1) sp = 1;
  long long ch = (keys + sp - 1) / sp;
  ch = (ch + kDecBlk - 1) / kDecBlk * kDecBlk;
  sp = (keys + ch - 1) / ch;
  *mt = m;
  *splits = static_cast<int>(sp);
  *chunk = static_cast<int>(ch);
}

cudaError_t launch_decode(const DecodeParams& p, cudaStream_t stream) {
  if (p.D == 64) return launch_decode_d<64>(p, stream);
  if (p.D == 128) return launch_decode_d<128>(p, stream);
  return cudaErrorInvalidValue;
}

}  // namespace hd
