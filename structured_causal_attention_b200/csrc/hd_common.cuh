// hd_common.cuh - shared device helpers for the Hidden Decoding kernels (sm_100a).
//
// Layout conventions (expanded sequence of the page "微信WeLM提出Hidden Decoding：
// 大模型推理新范式", section "隐式序列缩放的技术细节", step 1, 0-based):
// position p = t*n + s holds stream s of token t.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/hd.h"

namespace hd {

// ---------------------------------------------------------------- status word
// One int per device, owned by api.cu; kernels receive its address and record
// the first error code with atomicCAS (never trap).
__device__ __forceinline__ void record_status(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

// Bounds check of a computed index, compiled in only in the checked build
// (HD_CHECK_BOUNDS): an access of elements [i, i + n) of a buffer of `ext`
// elements that does not fit records HD_ERR_DEVICE_INDEX and returns false, and
// the caller skips the access. In the normal build it is constant true and
// costs nothing.
__device__ __forceinline__ bool in_bounds(long long i, long long n, long long ext, int* status) {
#ifdef HD_CHECK_BOUNDS
  if (i >= 0 && n >= 0 && i + n <= ext) return true;
  record_status(status, HD_ERR_DEVICE_INDEX);
  return false;
#else
  (void)i; (void)n; (void)ext; (void)status;
  return true;
#endif
}

// ------------------------------------------------------------- attention problem
// One attention "problem" is a (batch, query head, stream-group) triple whose
// query rows r = 0..Lq-1 and key rows c = 0..Lk-1 are addressed with constant
// strides. Key c is visible from row r iff
//     c <= a*r + bb   and   c > a*r + bb - win
// which covers every mode:
//   INTRA (de-interleaved stream s): a=1, bb=0, win=INF, rows/keys stride n
//   CROSS_FULL:                     a=1, bb=0, win=INF
//   CROSS_WINDOW:                   a=1, bb=0, win=n*W
//   final-stream-only CROSS_*:      a=n, bb=n-1 (row t is position t*n+n-1)
//   final-stream-only INTRA:        a=1, bb=0 on stream n-1's keys
struct AttnParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  __nv_bfloat16* o;
  float* lse;
  // backward only
  const __nv_bfloat16* dout;
  float* dq_acc;        // fp32 accumulator, q's layout
  float* lse2p;         // LSE * log2(e), packed per problem: [B][Hq][groups][lq_pad]
  float* deltap;        // rowsum(dO * O), same packed layout
  int lq_pad;           // Lq rounded up to 64 (padding rows hold zeros)
  __nv_bfloat16* dq;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  int* status;

  int B, Hq, Hkv, D, n, L, S, Sq;  // Sq = rows of q per batch in memory (S or L)
  int mode, final_only;
  int groups;           // independent stream groups per (b, h): n for INTRA, else 1
  int Lq, Lk;           // query rows / keys per problem
  int a, bb, win;       // visibility rule (see above)
  int qs_step;          // memory row offset of group s = s * qs_step (q, o, lse rows)
  int ks_step;          // memory row offset of group s for k, v
  int ks_base;          // extra key row offset (n-1 for final-only INTRA)
  int q_rstride;        // memory rows between consecutive problem rows (1 or n)
  int k_rstride;
  float scale;
  float scale_log2;     // scale * log2(e)
  // allocated elements, for the checked build's bounds checks
  long long ext_q;      // q, out, dout, dq, dq_acc: B * Sq * Hq * D
  long long ext_lse;    // lse: B * Hq * Sq
  long long ext_kv;     // k, v, dk, dv: B * S * Hkv * D
  long long ext_packed; // lse2p, deltap: packed rows
};

__device__ __forceinline__ bool key_visible(const AttnParams& p, int r, int c) {
  const int hi = p.a * r + p.bb;
  return c <= hi && c > hi - p.win && c < p.Lk;
}

// ------------------------------------------------------------------ PTX helpers
__device__ __forceinline__ uint32_t smem_u32(const void* ptr) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(ptr));
}

// 16-byte async copy global -> shared; src_bytes = 0 zero-fills the destination.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src),
               "r"(src_bytes));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// D(16x8 fp32) += A(16x16 bf16, row) * B(16x8 bf16, col)
__device__ __forceinline__ void mma_bf16_16816(float* d, const uint32_t* a, uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Two fp32 values as one 64-bit register pair (low half first).
__device__ __forceinline__ uint64_t pack_f32x2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}

// (y0, y1) = (a0, a1) * b + c on both halves of a register pair with one
// paired FMA (sm_100 fma.rn.f32x2); each half rounds exactly like fmaf. a0
// and a1 are fp32 bit patterns.
__device__ __forceinline__ void fma_f32x2(uint32_t a0, uint32_t a1, uint64_t b, uint64_t c, float& y0,
                                          float& y1) {
  uint64_t a, y;
  asm("mov.b64 %0, {%1, %2};" : "=l"(a) : "r"(a0), "r"(a1));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(y) : "l"(a), "l"(b), "l"(c));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(y0), "=f"(y1) : "l"(y));
}

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

// Swizzled offset (in bytes) of the 16-byte chunk `chunk` of row `row` in a tile
// whose rows are `row_chunks` chunks long: chunk index XOR (row % 8), so the 8
// rows an ldmatrix phase reads fall in 8 different bank groups.
__device__ __forceinline__ uint32_t swz(int row, int chunk, int row_chunks) {
  return static_cast<uint32_t>((row * row_chunks + (chunk ^ (row & 7))) * 16);
}

}  // namespace hd
