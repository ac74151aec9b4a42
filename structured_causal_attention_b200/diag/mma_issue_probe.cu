// mma_issue_probe.cu - how fast tcgen05.mma instructions can be issued.
//
// One CTA on one SM. NW warps each issue NMMA/NW back-to-back
// tcgen05.mma.cta_group::1.kind::f16 (M=128, N, K=16, both operands from
// zeroed shared memory) into their own TMEM columns, then commit to their own
// mbarrier; the probe prints the cycles from a common start to the last
// completion, per MMA, next to the MMA's run time at the nominal dense rate
// (8192 FLOP per cycle per SM). Two ways to issue: lane 0 alone runs the loop
// (WARP = 0), or the whole warp runs it with warp-uniform operands and one
// elected lane issues (WARP = 1). A diagnostic, not part of libhd.so:
//
//   nvcc -gencode arch=compute_100a,code=sm_100a -O3 -std=c++17 \
//        -I structured_causal_attention_b200/csrc \
//        -o mma_issue_probe structured_causal_attention_b200/diag/mma_issue_probe.cu
//   ./mma_issue_probe
#include <cstdint>
#include <cstdio>

#include "tc_ptx.cuh"

using namespace hd;

template <int N, int NW, int NMMA, int WARP>
__global__ void __launch_bounds__(128, 1) probe(long long* out, int* status) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - smem_u32(smem_raw));
  const uint32_t sA = sbase, sB = sbase + 16384;  // A: 128 x 64 bf16, B: N x 64 bf16
  const uint32_t bars = sbase + 16384 + N * 128;  // NW mbarriers
  const uint32_t slot = bars + 8 * NW;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sgen + (slot - sbase) + 4);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int i = tid; i < (16384 + N * 128) / 16; i += 128)
    asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};\n" ::"r"(sbase + i * 16), "r"(0) : "memory");
  tc::fence_async_smem();
  if (tid == 0) {
    for (int w = 0; w < NW; ++w) tc::mbar_init(bars + 8 * w, 1);
    *abort_flag = 0;
    tc::fence_mbar_init();
  }
  if (warp == 0) {
    tc::tmem_alloc(slot, 512);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sgen + (slot - sbase));
  const long long t0 = clock64();
  constexpr uint32_t id = tc::idesc_bf16_f32(128, N, 0, 0);
  if (WARP == 0) {
    if (warp < NW && lane == 0) {
      const uint64_t da = tc::smem_desc_sw128(sA, 16, 1024), db = tc::smem_desc_sw128(sB, 16, 1024);
#pragma unroll 1
      for (int i = 0; i < NMMA / NW; ++i) {
        const uint32_t kk = i & 3;
        tc::mma_ss(tmem + warp * N, da + ((kk * 32) >> 4), db + ((kk * 32) >> 4), id, i > 0);
      }
      tc::mma_commit(bars + 8 * warp);
      tc::mbar_wait(bars + 8 * warp, 0, abort_flag, status);
      out[warp] = clock64() - t0;
    }
  } else if (warp < NW) {
    const uint64_t da = tc::smem_desc_sw128(sA, 16, 1024), db = tc::smem_desc_sw128(sB, 16, 1024);
#pragma unroll 8
    for (int i = 0; i < NMMA / NW; ++i) {
      const uint32_t kk = i & 3;
      tc::mma_ss_elect(tmem + warp * N, da + ((kk * 32) >> 4), db + ((kk * 32) >> 4), id, i > 0);
    }
    tc::mma_commit_elect(bars + 8 * warp);
    if (lane == 0) {
      tc::mbar_wait(bars + 8 * warp, 0, abort_flag, status);
      out[warp] = clock64() - t0;
    }
    __syncwarp();
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, 512);
  }
}

template <int N, int NW, int NMMA, int WARP>
void run(long long* d_out, int* d_st) {
  static_assert(N * NW <= 512, "TMEM columns");
  const int smem = 16384 + N * 128 + 8 * NW + 64 + 1024;
  cudaFuncSetAttribute(probe<N, NW, NMMA, WARP>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  for (int rep = 0; rep < 3; ++rep) {
    probe<N, NW, NMMA, WARP><<<1, 128, smem>>>(d_out, d_st);
    long long h[4] = {0, 0, 0, 0};
    if (cudaMemcpy(h, d_out, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) {
      printf("CUDA error\n");
      return;
    }
    long long mx = 0;
    for (int w = 0; w < NW; ++w) mx = h[w] > mx ? h[w] : mx;
    if (rep == 2)
      printf("N=%3d issuing warps=%d issue=%s  %6.1f cycles per MMA  (run time %3d)\n", N, NW,
             WARP ? "warp-wide" : "lane 0   ",
             static_cast<double>(mx) / NMMA, 128 * N * 16 * 2 / 8192);
  }
}

int main() {
  long long* d_out;
  int* d_st;
  cudaMalloc(&d_out, 64);
  cudaMalloc(&d_st, 4);
  cudaMemset(d_st, 0, 4);
  run<64, 1, 512, 0>(d_out, d_st);
  run<64, 2, 512, 0>(d_out, d_st);
  run<128, 1, 512, 0>(d_out, d_st);
  run<128, 2, 512, 0>(d_out, d_st);
  run<256, 1, 512, 0>(d_out, d_st);
  run<64, 1, 512, 1>(d_out, d_st);
  run<64, 2, 512, 1>(d_out, d_st);
  run<128, 1, 512, 1>(d_out, d_st);
  run<128, 2, 512, 1>(d_out, d_st);
  run<256, 1, 512, 1>(d_out, d_st);
  int st = 0;
  cudaMemcpy(&st, d_st, 4, cudaMemcpyDeviceToHost);
  printf("device status %d (0 = every wait completed)\n", st);
  return 0;
}
