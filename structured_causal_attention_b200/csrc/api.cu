// api.cu - the C ABI declared in include/hd.h: argument validation, problem
// set-up, launches. Everything is enqueued on the caller's stream; nothing is
// allocated.
#include <math.h>

#include <cmath>

#include "hd_common.cuh"
#include "launch.h"

namespace hd {

// Per-device status word: kernels record the first error code here.
__device__ int g_status_word;

namespace {

// Device address of the status word on the current device. Host code must not
// pass the symbol itself to a kernel: it names a host-side stand-in. The
// address is looked up on every call (a map lookup in the runtime), so it is
// never stale, not even after the device was reset.
int* status_ptr() {
  void* ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_status_word) != cudaSuccess) return nullptr;
  return static_cast<int*>(ptr);
}

bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

constexpr long long kMaxPositions = 1LL << 28;  // positions and rows stay far below kWinInf

int check_attn(const void* q, const void* k, const void* v, int B, int L, int n, int Hq, int Hkv,
               int D, int mode, int W, int final_only, float scale) {
  if (!q || !k || !v) return HD_ERR_INVALID_ARG;
  if (B < 1 || L < 1 || n < 1 || Hq < 1 || Hkv < 1 || D < 1) return HD_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return HD_ERR_INVALID_ARG;
  if (mode < HD_INTRA || mode > HD_CROSS_WINDOW) return HD_ERR_INVALID_ARG;
  if (mode == HD_CROSS_WINDOW && W < 1) return HD_ERR_INVALID_ARG;
  if (final_only != 0 && final_only != 1) return HD_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !isfinite(scale)) return HD_ERR_INVALID_ARG;
  if (static_cast<long long>(n) * L > kMaxPositions) return HD_ERR_UNSUPPORTED;
  if (D != 64 && D != 128) return HD_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v)) return HD_ERR_INVALID_ARG;
  return HD_OK;
}

// Streaming multiprocessors of the current device; 148 (a B200) when no device
// can be queried, so that workspace sizes can still be computed without one.
int sm_count() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1) {
    cudaGetLastError();  // clear the error the failed query recorded
    return 148;
  }
  return sms;
}

AttnParams make_params(const void* q, const void* k, const void* v, int B, int L, int n, int Hq,
                       int Hkv, int D, int mode, int W, int final_only, float scale) {
  AttnParams p = {};
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k = static_cast<const __nv_bfloat16*>(k);
  p.v = static_cast<const __nv_bfloat16*>(v);
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.D = D;
  p.n = n;
  p.L = L;
  p.S = n * L;
  p.Sq = final_only ? L : n * L;
  p.mode = mode;
  p.final_only = final_only;
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634074f;
  p.status = status_ptr();
  p.ext_q = static_cast<long long>(B) * p.Sq * Hq * D;
  p.ext_lse = static_cast<long long>(B) * Hq * p.Sq;
  p.ext_kv = static_cast<long long>(B) * p.S * Hkv * D;
  if (mode == HD_INTRA) {
    // each stream is its own causal problem over the L tokens
    p.groups = final_only ? 1 : n;
    p.Lq = L;
    p.Lk = L;
    p.a = 1;
    p.bb = 0;
    p.win = kWinInf;
    p.qs_step = final_only ? 0 : 1;
    p.ks_step = final_only ? 0 : 1;
    p.ks_base = final_only ? n - 1 : 0;
    p.q_rstride = final_only ? 1 : n;
    p.k_rstride = n;
  } else {
    p.groups = 1;
    p.Lq = p.Sq;
    p.Lk = p.S;
    p.a = final_only ? n : 1;
    p.bb = final_only ? n - 1 : 0;
    const long long w = static_cast<long long>(n) * W;
    p.win = (mode == HD_CROSS_WINDOW && w < p.S) ? static_cast<int>(w) : kWinInf;
    p.qs_step = 0;
    p.ks_step = 0;
    p.ks_base = 0;
    p.q_rstride = 1;
    p.k_rstride = 1;
  }
  return p;
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

size_t pad64(size_t x) { return (x + 63) / 64 * 64; }

// Rows of the packed per-problem statistics (LSE, D) for any mode: each
// problem's rows are padded to a multiple of 64.
size_t packed_rows(int B, int L, int n, int Hq, int final_only) {
  // n * pad64(L) >= pad64(n * L): covers the n INTRA streams and the single
  // cross-stream problem alike
  const size_t per_bh = final_only ? pad64(L) : static_cast<size_t>(n) * pad64(L);
  return static_cast<size_t>(B) * Hq * per_bh;
}

int from_cuda(cudaError_t e) { return e == cudaSuccess ? HD_OK : HD_ERR_CUDA; }


// Split-K partials for `rows` query rows per (sequence, KV head) against up to
// `keys` keys: unnormalised O (fp32 [.., D]) and (max, sum) pairs.
size_t decode_partials_bytes(int B, int rows, long long keys, int Hkv, int D) {
  int mt = 0, splits = 0, chunk = 0;
  decode_split_plan(B, rows, keys, Hkv, sm_count(), &mt, &splits, &chunk);
  const size_t prow = static_cast<size_t>(B) * Hkv * mt * 16 * splits;
  return align256(prow * static_cast<size_t>(D) * 4) + align256(prow * 2 * 4);
}

// Workspace of one decode call. All n streams: n*g rows over the whole cache.
// Final stream alone: g rows over the whole cache (CROSS modes) or over its
// own Tcap rows (INTRA); the workspace covers both, so it does not depend on
// the mode.
size_t decode_workspace(int B, int n, int Tcap, int Hq, int Hkv, int D, int final_only) {
  if (B < 1 || n < 1 || Tcap < 1 || Hq < 1 || Hkv < 1 || D < 1 || Hq % Hkv) return 0;
  const int g = Hq / Hkv;
  const long long keys = static_cast<long long>(Tcap) * n;
  if (!final_only) return decode_partials_bytes(B, n * g, keys, Hkv, D);
  const size_t a = decode_partials_bytes(B, g, keys, Hkv, D);
  const size_t b = decode_partials_bytes(B, g, Tcap, Hkv, D);
  return a > b ? a : b;
}

int decode_call(const void* q, const void* k_cache, const void* v_cache, const int32_t* seqlen,
                void* out, float* lse, int B, int n, int Tcap, int Hq, int Hkv, int D, int mode,
                int W_tokens, int final_only, float scale, void* workspace,
                size_t workspace_bytes, void* stream) {
  if (!q || !k_cache || !v_cache || !seqlen || !out || !lse || !workspace) return HD_ERR_INVALID_ARG;
  if (B < 1 || n < 1 || Tcap < 1 || Hq < 1 || Hkv < 1 || D < 1) return HD_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return HD_ERR_INVALID_ARG;
  if (mode < HD_INTRA || mode > HD_CROSS_WINDOW) return HD_ERR_INVALID_ARG;
  if (mode == HD_CROSS_WINDOW && W_tokens < 1) return HD_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !isfinite(scale)) return HD_ERR_INVALID_ARG;
  if (static_cast<long long>(Tcap) * n > kMaxPositions) return HD_ERR_UNSUPPORTED;
  if (D != 64 && D != 128) return HD_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) ||
      !aligned16(workspace))
    return HD_ERR_INVALID_ARG;
  const size_t need = decode_workspace(B, n, Tcap, Hq, Hkv, D, final_only);
  if (workspace_bytes < need) return HD_ERR_INVALID_ARG;
  DecodeParams p = {};
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.kc = static_cast<const __nv_bfloat16*>(k_cache);
  p.vc = static_cast<const __nv_bfloat16*>(v_cache);
  p.seqlen = seqlen;
  p.o = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.status = status_ptr();
  p.B = B;
  p.n = n;
  p.Tcap = Tcap;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.D = D;
  p.mode = mode;
  const long long w = static_cast<long long>(n) * W_tokens;
  p.win = (mode == HD_CROSS_WINDOW && w < static_cast<long long>(Tcap) * n) ? static_cast<int>(w)
                                                                           : kWinInf;
  if (mode == HD_CROSS_WINDOW && p.win == kWinInf) p.mode = HD_CROSS_FULL;
  p.nq = final_only ? 1 : n;
  p.s0 = final_only ? n - 1 : 0;
  p.kstride = 1;
  p.kres = 0;
  p.kpt = n;
  if (final_only && mode == HD_INTRA && n > 1) {
    // the final stream's own rows only; each of them is visible to its query
    p.kstride = n;
    p.kres = n - 1;
    p.kpt = 1;
    p.mode = HD_CROSS_FULL;
  }
  p.rows = p.nq * (Hq / Hkv);
  decode_split_plan(B, p.rows, static_cast<long long>(Tcap) * p.kpt, Hkv, sm_count(), &p.mt,
                    &p.splits, &p.chunk);
  const size_t prow = static_cast<size_t>(B) * Hkv * p.mt * 16 * p.splits;
  p.ext_q = static_cast<long long>(B) * p.nq * Hq * D;
  p.ext_lse = static_cast<long long>(B) * Hq * p.nq;
  p.ext_cache = static_cast<long long>(B) * Tcap * n * Hkv * D;
  p.ext_part = static_cast<long long>(prow);
  p.part_o = static_cast<float*>(workspace);
  p.part_ml = reinterpret_cast<float*>(static_cast<char*>(workspace) + align256(prow * D * 4));
  p.scale_log2 = scale * 1.4426950408889634074f;
  return from_cuda(launch_decode(p, static_cast<cudaStream_t>(stream)));
}

}  // namespace
}  // namespace hd

using namespace hd;

extern "C" {

const char* hd_status_string(int status) {
  switch (status) {
    case HD_OK: return "HD_OK";
    case HD_ERR_INVALID_ARG: return "HD_ERR_INVALID_ARG: invalid argument";
    case HD_ERR_UNSUPPORTED: return "HD_ERR_UNSUPPORTED: sizes not supported by this build";
    case HD_ERR_CUDA: return "HD_ERR_CUDA: a CUDA call or launch failed";
    case HD_ERR_TIMEOUT: return "HD_ERR_TIMEOUT: a bounded wait on the device gave up";
    case HD_ERR_DEVICE_INDEX: return "HD_ERR_DEVICE_INDEX: an index read on the device was out of range";
    default: return "unknown hd_status";
  }
}

int hd_version(void) { return (1 << 16) | 2; }

int hd_build_flags(void) {
#ifdef HD_CHECK_BOUNDS
  return HD_BUILD_CHECK_BOUNDS;
#else
  return 0;
#endif
}

int hd_expand_embed(const int32_t* ids, const void* tables, void* out, int B, int L, int n, int V,
                    int d, int elem_bytes, void* stream) {
  if (!ids || !tables || !out) return HD_ERR_INVALID_ARG;
  if (B < 1 || L < 1 || n < 1 || V < 1 || d < 1) return HD_ERR_INVALID_ARG;
  if (elem_bytes != 1 && elem_bytes != 2 && elem_bytes != 4 && elem_bytes != 8)
    return HD_ERR_INVALID_ARG;
  const long long row_bytes = static_cast<long long>(d) * elem_bytes;
  if (elem_bytes == 1 && row_bytes % 2 != 0) return HD_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(tables) | reinterpret_cast<uintptr_t>(out)) % 2 != 0)
    return HD_ERR_INVALID_ARG;
  return from_cuda(launch_expand(ids, tables, out, B, L, n, V, row_bytes, sm_count(), status_ptr(),
                                 static_cast<cudaStream_t>(stream)));
}

int hd_rope_expanded(void* q, void* k, const int32_t* token_offset, int B, int L, int n, int Hq,
                     int Hkv, int D, int final_stream_queries_only, double base, void* stream) {
  if (!q && !k) return HD_ERR_INVALID_ARG;
  if (B < 1 || L < 1 || n < 1 || D < 1) return HD_ERR_INVALID_ARG;
  if ((q && Hq < 1) || (k && Hkv < 1)) return HD_ERR_INVALID_ARG;
  if (final_stream_queries_only != 0 && final_stream_queries_only != 1) return HD_ERR_INVALID_ARG;
  if (!(base > 1.0) || !std::isfinite(base)) return HD_ERR_INVALID_ARG;
  if ((q && !aligned16(q)) || (k && !aligned16(k))) return HD_ERR_INVALID_ARG;
  if (D != 16 && D != 32 && D != 64 && D != 128 && D != 256) return HD_ERR_UNSUPPORTED;
  if (static_cast<long long>(n) * L > (1LL << 30)) return HD_ERR_UNSUPPORTED;
  RopeParams p{};
  p.q = static_cast<__nv_bfloat16*>(q);
  p.k = static_cast<__nv_bfloat16*>(k);
  p.token_offset = token_offset;
  p.status = status_ptr();
  p.B = B;
  p.S = n * L;
  p.Sq = final_stream_queries_only ? L : n * L;
  p.n = n;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.D = D;
  p.final_only = final_stream_queries_only;
  p.log2_base = std::log2(base);
  return from_cuda(launch_rope(p, sm_count(), static_cast<cudaStream_t>(stream)));
}

int hd_final_readout(const void* x, void* out, int B, int L, int n, int d, int elem_bytes,
                     void* stream) {
  if (!x || !out) return HD_ERR_INVALID_ARG;
  if (B < 1 || L < 1 || n < 1 || d < 1) return HD_ERR_INVALID_ARG;
  if (elem_bytes != 1 && elem_bytes != 2 && elem_bytes != 4 && elem_bytes != 8)
    return HD_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(out)) return HD_ERR_INVALID_ARG;
  const long long row_bytes = static_cast<long long>(d) * elem_bytes;
  if (row_bytes % 16 != 0) return HD_ERR_UNSUPPORTED;
  return from_cuda(launch_final_readout(x, out, static_cast<long long>(B) * L, n, row_bytes, sm_count(),
                                        status_ptr(), static_cast<cudaStream_t>(stream)));
}

size_t hd_lm_head_ce_workspace_bytes(int B, int L, int V) {
  if (B < 1 || L < 1 || V < 1) return 0;
  return lm_head_workspace_bytes(static_cast<long long>(B) * L, V);
}

int hd_lm_head_ce(const void* x, const void* w, const int32_t* labels, float* loss, float* lse,
                  int B, int L, int n, int d, int V, void* workspace, size_t workspace_bytes,
                  void* stream) {
  if (!x || !w || !labels || !loss || !workspace) return HD_ERR_INVALID_ARG;
  if (B < 1 || L < 1 || n < 1 || d < 1 || V < 1) return HD_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w) || !aligned16(workspace)) return HD_ERR_INVALID_ARG;
  if (d % 64 != 0) return HD_ERR_UNSUPPORTED;
  const long long R = static_cast<long long>(B) * L;
  if (R > (1LL << 31) - 1) return HD_ERR_UNSUPPORTED;
  if (workspace_bytes < lm_head_workspace_bytes(R, V)) return HD_ERR_INVALID_ARG;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1)
    return HD_ERR_CUDA;
  LmHeadParams p{};
  p.labels = labels;
  p.loss = loss;
  p.lse = lse;
  p.R = R;
  p.V = V;
  p.d = d;
  const long long nvt = (V + 255) / 256;
  p.part = static_cast<float*>(workspace);
  p.pick = reinterpret_cast<float*>(static_cast<char*>(workspace) + align256(static_cast<size_t>(2 * nvt * R) * 4));
  p.status = status_ptr();
  return from_cuda(launch_lm_head_ce(p, x, w, n, sms, static_cast<cudaStream_t>(stream)));
}

size_t hd_lm_head_ce_bwd_workspace_bytes(int B, int L, int V) {
  if (B < 1 || L < 1 || V < 1) return 0;
  return lm_head_grad_workspace_bytes(static_cast<long long>(B) * L, V);
}

int hd_lm_head_ce_bwd(const void* x, const void* w, const int32_t* labels, const float* lse,
                      float grad_scale, void* dh, float* dw, int B, int L, int n, int d, int V,
                      void* workspace, size_t workspace_bytes, void* stream) {
  if (!x || !w || !labels || !lse || !dh || !dw || !workspace) return HD_ERR_INVALID_ARG;
  if (B < 1 || L < 1 || n < 1 || d < 1 || V < 1) return HD_ERR_INVALID_ARG;
  if (!std::isfinite(grad_scale)) return HD_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w) || !aligned16(dh) || !aligned16(dw) || !aligned16(workspace))
    return HD_ERR_INVALID_ARG;
  if (d % 64 != 0) return HD_ERR_UNSUPPORTED;
  const long long R = static_cast<long long>(B) * L;
  if (R > (1LL << 31) - 1) return HD_ERR_UNSUPPORTED;
  if (workspace_bytes < lm_head_grad_workspace_bytes(R, V)) return HD_ERR_INVALID_ARG;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1)
    return HD_ERR_CUDA;
  LmHeadParams p{};
  p.labels = labels;
  p.lse_in = lse;
  p.g = static_cast<__nv_bfloat16*>(workspace);
  p.R = R;
  p.V = V;
  p.d = d;
  p.status = status_ptr();
  return from_cuda(launch_lm_head_ce_bwd(p, x, w, n, grad_scale, dh, dw, sms,
                                         static_cast<cudaStream_t>(stream)));
}

int hd_attn_fwd(const void* q, const void* k, const void* v, void* out, float* lse, int B, int L,
                int n, int Hq, int Hkv, int D, int mode, int W_tokens,
                int final_stream_queries_only, float scale, void* stream) {
  int st = check_attn(q, k, v, B, L, n, Hq, Hkv, D, mode, W_tokens, final_stream_queries_only, scale);
  if (st != HD_OK) return st;
  if (!out || !lse || !aligned16(out)) return HD_ERR_INVALID_ARG;
  AttnParams p = make_params(q, k, v, B, L, n, Hq, Hkv, D, mode, W_tokens,
                             final_stream_queries_only, scale);
  p.o = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  return from_cuda(launch_attn_fwd_tc(p, static_cast<cudaStream_t>(stream)));
}

size_t hd_attn_bwd_workspace_bytes(int B, int L, int n, int Hq, int Hkv, int D,
                                   int final_stream_queries_only) {
  if (B < 1 || L < 1 || n < 1 || Hq < 1 || Hkv < 1 || D < 1) return 0;
  const size_t Sq = final_stream_queries_only ? static_cast<size_t>(L)
                                              : static_cast<size_t>(n) * static_cast<size_t>(L);
  const size_t rows = static_cast<size_t>(B) * Sq * static_cast<size_t>(Hq);
  return align256(rows * static_cast<size_t>(D) * 4) + 2 * align256(packed_rows(B, L, n, Hq, final_stream_queries_only) * 4);
}

int hd_attn_bwd(const void* q, const void* k, const void* v, const void* out, const float* lse,
                const void* dout, void* dq, void* dk, void* dv, int B, int L, int n, int Hq,
                int Hkv, int D, int mode, int W_tokens, int final_stream_queries_only,
                float scale, void* workspace, size_t workspace_bytes, void* stream) {
  int st = check_attn(q, k, v, B, L, n, Hq, Hkv, D, mode, W_tokens, final_stream_queries_only, scale);
  if (st != HD_OK) return st;
  if (!out || !lse || !dout || !dq || !dk || !dv || !workspace) return HD_ERR_INVALID_ARG;
  if (!aligned16(out) || !aligned16(dout) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv) ||
      !aligned16(workspace))
    return HD_ERR_INVALID_ARG;
  const size_t need = hd_attn_bwd_workspace_bytes(B, L, n, Hq, Hkv, D, final_stream_queries_only);
  if (workspace_bytes < need) return HD_ERR_INVALID_ARG;
  AttnParams p = make_params(q, k, v, B, L, n, Hq, Hkv, D, mode, W_tokens,
                             final_stream_queries_only, scale);
  p.o = static_cast<__nv_bfloat16*>(const_cast<void*>(out));
  p.lse = const_cast<float*>(lse);
  p.dout = static_cast<const __nv_bfloat16*>(dout);
  p.dq = static_cast<__nv_bfloat16*>(dq);
  p.dk = static_cast<__nv_bfloat16*>(dk);
  p.dv = static_cast<__nv_bfloat16*>(dv);
  const size_t rows = static_cast<size_t>(B) * p.Sq * Hq;
  p.dq_acc = static_cast<float*>(workspace);
  const size_t npk = packed_rows(B, L, n, Hq, final_stream_queries_only);
  p.lse2p = reinterpret_cast<float*>(static_cast<char*>(workspace) + align256(rows * D * 4));
  p.deltap = reinterpret_cast<float*>(reinterpret_cast<char*>(p.lse2p) + align256(npk * 4));
  p.lq_pad = static_cast<int>(pad64(p.Lq));
  p.ext_packed = static_cast<long long>(npk);
  return from_cuda(launch_attn_bwd(p, static_cast<cudaStream_t>(stream)));
}

size_t hd_decode_workspace_bytes(int B, int n, int Tcap, int Hq, int Hkv, int D) {
  return hd::decode_workspace(B, n, Tcap, Hq, Hkv, D, 0);
}

size_t hd_decode_final_workspace_bytes(int B, int n, int Tcap, int Hq, int Hkv, int D) {
  return hd::decode_workspace(B, n, Tcap, Hq, Hkv, D, 1);
}

int hd_decode_attn(const void* q, const void* k_cache, const void* v_cache, const int32_t* seqlen,
                   void* out, float* lse, int B, int n, int Tcap, int Hq, int Hkv, int D, int mode,
                   int W_tokens, float scale, void* workspace, size_t workspace_bytes,
                   void* stream) {
  return hd::decode_call(q, k_cache, v_cache, seqlen, out, lse, B, n, Tcap, Hq, Hkv, D, mode,
                         W_tokens, 0, scale, workspace, workspace_bytes, stream);
}

int hd_decode_attn_final(const void* q, const void* k_cache, const void* v_cache,
                         const int32_t* seqlen, void* out, float* lse, int B, int n, int Tcap,
                         int Hq, int Hkv, int D, int mode, int W_tokens, float scale,
                         void* workspace, size_t workspace_bytes, void* stream) {
  return hd::decode_call(q, k_cache, v_cache, seqlen, out, lse, B, n, Tcap, Hq, Hkv, D, mode,
                         W_tokens, 1, scale, workspace, workspace_bytes, stream);
}

int hd_selftest_wait_timeout(long long limit_cycles, void* stream) {
  if (limit_cycles < 1 || limit_cycles > (1LL << 33)) return HD_ERR_INVALID_ARG;
  return from_cuda(launch_wait_timeout(limit_cycles, status_ptr(), static_cast<cudaStream_t>(stream)));
}

int hd_device_status(void* stream, int clear) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return HD_ERR_CUDA;
  int* ptr = status_ptr();
  if (!ptr) return HD_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, ptr, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return HD_ERR_CUDA;
  if (clear && v != 0) {
    const int zero = 0;
    if (cudaMemcpy(ptr, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return HD_ERR_CUDA;
  }
  return v;
}

}  // extern "C"
