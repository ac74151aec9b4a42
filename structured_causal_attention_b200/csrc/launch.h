// launch.h - internal host launchers (not part of the C ABI).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "hd_common.cuh"

namespace hd {

constexpr int kWinInf = 1 << 30;  // "no window": larger than any supported sequence

cudaError_t launch_attn_fwd_tc(const AttnParams& p, cudaStream_t stream);
cudaError_t launch_attn_bwd(const AttnParams& p, cudaStream_t stream);
cudaError_t launch_attn_bwd_tc_main(const AttnParams& p, cudaStream_t stream);

struct DecodeParams {
  const __nv_bfloat16* q;   // [B, nq, Hq, D]
  const __nv_bfloat16* kc;  // [B, Tcap*n, Hkv, D]
  const __nv_bfloat16* vc;
  const int32_t* seqlen;    // [B]
  __nv_bfloat16* o;         // [B, nq, Hq, D]
  float* lse;               // [B, Hq, nq]
  float* part_o;            // [B, Hkv, MT*16, splits, D] fp32
  float* part_ml;           // [B, Hkv, MT*16, splits, 2] fp32 (max in log2 units, sum)
  int* status;
  int B, n, Tcap, Hq, Hkv, D, mode, win;  // win = n*W or kWinInf
  // Query streams s0 .. s0+nq-1 of the new token (all n, or only the final one).
  int nq, s0;
  // Keys are indexed in a "key space": key index c is cache position
  // kres + c*kstride, and a sequence of T1 tokens holds T1*kpt keys. The whole
  // cache: (1, 0, n). The final stream alone (final-stream-only INTRA): (n, n-1, 1).
  int kstride, kres, kpt;
  int rows, mt, splits, chunk;             // rows = nq*(Hq/Hkv); chunk keys per split
  float scale_log2;
  // allocated elements, for the checked build's bounds checks
  long long ext_q;      // q, o: B * nq * Hq * D
  long long ext_lse;    // lse: B * Hq * nq
  long long ext_cache;  // each cache: B * Tcap * n * Hkv * D
  long long ext_part;   // partial rows: B * Hkv * mt * 16 * splits
};

// Number of splits / chunk length the decode launcher uses for `rows` query
// rows per (sequence, KV head) against up to `keys` keys on a GPU of `sms`
// streaming multiprocessors.
void decode_split_plan(int B, int rows, long long keys, int Hkv, int sms, int* mt, int* splits,
                       int* chunk);
cudaError_t launch_decode(const DecodeParams& p, cudaStream_t stream);

struct RopeParams {
  __nv_bfloat16* q;             // [B, Sq, Hq, D] or null
  __nv_bfloat16* k;             // [B, S, Hkv, D] or null
  const int32_t* token_offset;  // [B] tokens before the call, or null (all 0)
  int* status;
  int B, S, Sq, n, Hq, Hkv, D, final_only;
  double log2_base;
};
cudaError_t launch_rope(const RopeParams& p, int sms, cudaStream_t stream);

struct LmHeadParams {
  const int32_t* labels;  // [R]
  float* loss;            // [R]
  float* lse;             // [R] or null
  float* part;            // [2][nvt][R]: per vocabulary tile max (log2 units), sum of exp2
  float* pick;            // [R] logit of the label
  int* status;
  long long R;            // rows (tokens) = B*L
  int V, d;
  int nrb, nvt;           // row pairs, vocabulary tiles (set by the launcher)
  long long units;
  // gradient pass only
  const float* lse_in;    // [R] natural-log LSE of the forward
  __nv_bfloat16* g;       // [R, g_ld] softmax - onehot, bf16
  long long g_ld;         // columns of g: V rounded up to 256
};
size_t lm_head_workspace_bytes(long long R, int V);
size_t lm_head_grad_workspace_bytes(long long R, int V);
cudaError_t launch_lm_head_ce_bwd(LmHeadParams p, const void* x, const void* w, int n, float scale,
                                  void* dh, float* dw, int num_sms, cudaStream_t stream);
cudaError_t launch_lm_head_ce(LmHeadParams p, const void* x, const void* w, int n, int num_sms,
                              cudaStream_t stream);
cudaError_t launch_final_readout(const void* x, void* out, long long rows, int n,
                                 long long row_bytes, int sms, int* status, cudaStream_t stream);

cudaError_t launch_wait_timeout(long long limit_cycles, int* status, cudaStream_t stream);

cudaError_t launch_expand(const int32_t* ids, const void* tables, void* out, int B, int L, int n,
                          int V, long long row_bytes, int sms, int* status, cudaStream_t stream);

}  // namespace hd
