// fa_api.cu -- the C ABI of libfa.so (declared in include/fa.h): argument
// checking, TMA descriptor construction and kernel launches.  Every entry point
// validates on the host first and enqueues nothing when an argument is bad.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <mutex>

#include "../../include/fa.h"
#include "bwd_sm100.cuh"
#include "fwd_sm100.cuh"
#include "simt_f32.cuh"

namespace {

constexpr int kAbiVersion = 100;

cudaEvent_t g_ev_start = nullptr, g_ev_stop = nullptr;  // fa_set_timing_events
inline void mark_start(cudaStream_t st) {
  if (g_ev_start && g_ev_stop) cudaEventRecord(g_ev_start, st);
}
inline void mark_stop(cudaStream_t st) {
  if (g_ev_start && g_ev_stop) cudaEventRecord(g_ev_stop, st);
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

fa_status check_common(int B, int H, int Hkv, int N, int d, float scale, int window, fa_dtype dtype) {
  if (B < 1 || H < 1 || Hkv < 1 || N < 1) return FA_ERR_INVALID_ARG;
  if (H % Hkv != 0) return FA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (window < -1) return FA_ERR_INVALID_ARG;
  if (dtype != FA_BF16 && dtype != FA_FP32) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  // Index arithmetic inside the kernels is 32-bit for rows of one head and for
  // the grid: keep every count well inside int range.
  if (static_cast<long long>(B) * H * ((N + 255) / 256) > 0x7fffffffLL) return FA_ERR_UNSUPPORTED;
  if (N > (1 << 30)) return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

inline size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

inline int padded_rows(int N) { return (N + 127) / 128 * 128; }

// ---------------------------------------------------------------- TMA descriptors
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// A [heads, N, d] bf16 tensor seen in 128-row x 64-column boxes with the
// 128-byte swizzle (the layout the UMMA descriptors expect).
bool make_tile_map(CUtensorMap* m, const void* ptr, int heads, int N, int d) {
  EncodeTiledFn enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(heads)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(N) * d * 2};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename K>
bool set_smem(K kernel, int bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) == cudaSuccess;
}

inline fa_status launched() { return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA; }

fa::SimtParams simt_params(int B, int H, int Hkv, int N, float scale, int causal, int window) {
  fa::SimtParams s{};
  s.B = B;
  s.H = H;
  s.Hkv = Hkv;
  s.N = N;
  s.g = H / Hkv;
  s.scale = scale;
  s.causal = causal ? 1 : 0;
  s.window = window;
  return s;
}

inline size_t splitkv_ws_bytes(int B, int H, int N, int d, int splits) {
  const size_t nq2 = static_cast<size_t>((N + 255) / 256) * 256;
  return align256(static_cast<size_t>(splits) * B * H * nq2 * d * 4) +
         align256(static_cast<size_t>(splits) * B * H * nq2 * 16);
}

// splits == 0: the plain forward; splits >= 1: split-KV partials into `ws`
// followed by the merge kernel.
template <int D>
fa_status fwd_bf16(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Hkv, int N,
                   float scale, int causal, int window, cudaStream_t st, int splits = 0, void* ws = nullptr,
                   const uint8_t* bmask = nullptr, long long bmask_hs = 0, const int* seqlens = nullptr) {
  using C = fa::FwdCfg<D>;
  CUtensorMap tq, tk, tv, to;
  if (!make_tile_map(&tq, q, B * H, N, D) || !make_tile_map(&tk, k, B * Hkv, N, D) ||
      !make_tile_map(&tv, v, B * Hkv, N, D) || !make_tile_map(&to, o, B * H, N, D))
    return FA_ERR_CUDA;
  if (!set_smem(fa::fwd_sm100_kernel<D, false, false>, C::kSmemBytes) ||
      !set_smem(fa::fwd_sm100_kernel<D, true, false>, C::kSmemBytes) ||
      !set_smem(fa::fwd_sm100_kernel<D, false, true>, C::kSmemBytes))
    return FA_ERR_CUDA;
  fa::FwdParams p{};
  p.lse = lse;
  p.B = B;
  p.H = H;
  p.Hkv = Hkv;
  p.N = N;
  p.g = H / Hkv;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.causal = causal ? 1 : 0;
  p.window = window;
  p.npairs = (N + 255) / 256;
  p.ntiles_kv = (N + 127) / 128;
  p.bmask = bmask;
  p.bmask_hs = bmask_hs;
  p.nbt = p.ntiles_kv;
  p.seqlens = seqlens;
  {  // heads per group: Q, O and the (shared) K, V of a group within ~64 MiB of L2
    const double unit = static_cast<double>(N) * D * (4.0 + 4.0 / p.g);
    p.group = std::min(B * H, static_cast<int>(std::max(1.0, std::floor((64.0 * 1024 * 1024) / unit))));
    p.group = std::max(p.g, p.group / p.g * p.g);  // whole GQA groups
    p.group = std::min(p.group, B * H);
  }
  const unsigned grid = static_cast<unsigned>(p.npairs) * B * H;
  if (splits == 0) {
    mark_start(st);
    if (bmask)
      fa::fwd_sm100_kernel<D, false, true><<<grid, C::kThreads, C::kSmemBytes, st>>>(tq, tk, tv, to, p);
    else
      fa::fwd_sm100_kernel<D, false, false><<<grid, C::kThreads, C::kSmemBytes, st>>>(tq, tk, tv, to, p);
    mark_stop(st);
    return launched();
  }
  p.splits = splits;
  p.nq2 = p.npairs * 256;
  p.part_o = static_cast<float*>(ws);
  p.part_m = reinterpret_cast<float4*>(static_cast<uint8_t*>(ws) +
                                       align256(static_cast<size_t>(splits) * B * H * p.nq2 * D * 4));
  mark_start(st);
  fa::fwd_sm100_kernel<D, true, false><<<grid * splits, C::kThreads, C::kSmemBytes, st>>>(tq, tk, tv, to, p);
  mark_stop(st);
  if (launched() != FA_OK) return FA_ERR_CUDA;
  const unsigned cgrid = static_cast<unsigned>(B * H) * ((N + 31) / 32);
  fa::fwd_combine_kernel<D><<<cgrid, 256, 0, st>>>(p, o);
  return launched();
}

template <int D>
fa_status fwd_f32(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Hkv, int N,
                  float scale, int causal, int window, cudaStream_t st, const uint8_t* bmask = nullptr,
                  long long bmask_hs = 0, const int* seqlens = nullptr) {
  fa::SimtParams s = simt_params(B, H, Hkv, N, scale, causal, window);
  s.bmask = bmask;
  s.bmask_hs = bmask_hs;
  s.nbt = (N + 127) / 128;
  s.seqlens = seqlens;
  s.q = static_cast<const float*>(q);
  s.k = static_cast<const float*>(k);
  s.v = static_cast<const float*>(v);
  s.o_out = static_cast<float*>(o);
  s.lse_out = lse;
  dim3 grid((N + fa::kSimtRows - 1) / fa::kSimtRows, B * H);
  mark_start(st);
  fa::fwd_simt_f32_kernel<D><<<grid, 32 * fa::kSimtRows, 0, st>>>(s);
  mark_stop(st);
  return launched();
}

struct WsLayout {
  size_t lse2, drow, dqacc, total;
};
WsLayout ws_layout(int B, int H, int N, int d, fa_dtype dtype) {
  WsLayout w{};
  if (dtype == FA_FP32) {
    w.drow = 0;
    w.total = align256(static_cast<size_t>(B) * H * N * 4);
    return w;
  }
  const size_t rows = static_cast<size_t>(B) * H * padded_rows(N);
  w.lse2 = 0;
  w.drow = align256(rows * 4);
  w.dqacc = w.drow + align256(rows * 4);
  w.total = w.dqacc + align256(rows * d * 4);
  return w;
}

template <int D>
fa_status bwd_bf16(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
                   void* dq, void* dk, void* dv, void* ws, int B, int H, int Hkv, int N, float scale, int causal,
                   int window, cudaStream_t st, const uint8_t* bmask = nullptr, long long bmask_hs = 0,
                   const int* seqlens = nullptr) {
  using C = fa::BwdCfg<D>;
  const WsLayout w = ws_layout(B, H, N, D, FA_BF16);
  uint8_t* wb = static_cast<uint8_t*>(ws);
  fa::BwdParams p{};
  p.lse = lse;
  p.o = o;
  p.dout = dout;
  p.lse2 = reinterpret_cast<float*>(wb + w.lse2);
  p.Drow = reinterpret_cast<float*>(wb + w.drow);
  p.dqacc = reinterpret_cast<float*>(wb + w.dqacc);
  p.dq = dq;
  p.B = B;
  p.H = H;
  p.Hkv = Hkv;
  p.N = N;
  p.Np = padded_rows(N);
  p.g = H / Hkv;
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.causal = causal ? 1 : 0;
  p.window = window;
  p.ntiles = p.Np / 128;
  p.bmask = bmask;
  p.bmask_hs = bmask_hs;
  p.seqlens = seqlens;
  // kv heads per rasterisation group: keep each group's Q, dO, K, V and dQ
  // accumulator (about N*d*(4 + 8g) bytes per kv head) within ~64 MiB of L2.
  {
    const double unit = static_cast<double>(p.Np) * D * (4.0 + 8.0 * p.g);
    p.group = static_cast<int>(std::max(1.0, std::floor((64.0 * 1024 * 1024) / unit)));
    p.group = std::min(p.group, B * Hkv);
  }
  CUtensorMap tq, tk, tv, tdo, tdk, tdv;
  if (!make_tile_map(&tq, q, B * H, N, D) || !make_tile_map(&tk, k, B * Hkv, N, D) ||
      !make_tile_map(&tv, v, B * Hkv, N, D) || !make_tile_map(&tdo, dout, B * H, N, D) ||
      !make_tile_map(&tdk, dk, B * Hkv, N, D) || !make_tile_map(&tdv, dv, B * Hkv, N, D))
    return FA_ERR_CUDA;
  if (!set_smem(fa::bwd_sm100_kernel<D, false>, C::kSmemBytes) ||
      !set_smem(fa::bwd_sm100_kernel<D, true>, C::kSmemBytes))
    return FA_ERR_CUDA;
  const size_t rows = static_cast<size_t>(B) * H * p.Np;
  fa::bwd_pre_kernel<D><<<static_cast<unsigned>((rows + 7) / 8), 256, 0, st>>>(p);
  if (launched() != FA_OK) return FA_ERR_CUDA;
  const unsigned grid = static_cast<unsigned>(p.ntiles) * B * Hkv;
  mark_start(st);
  if (bmask)
    fa::bwd_sm100_kernel<D, true><<<grid, C::kThreads, C::kSmemBytes, st>>>(tq, tk, tv, tdo, tdk, tdv, p);
  else
    fa::bwd_sm100_kernel<D, false><<<grid, C::kThreads, C::kSmemBytes, st>>>(tq, tk, tv, tdo, tdk, tdv, p);
  mark_stop(st);
  if (launched() != FA_OK) return FA_ERR_CUDA;
  fa::bwd_dq_kernel<D><<<static_cast<unsigned>(static_cast<size_t>(B) * H * (p.Np / 32)), 256, 0, st>>>(p);
  return launched();
}

template <int D>
fa_status bwd_f32(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
                  void* dq, void* dk, void* dv, void* ws, int B, int H, int Hkv, int N, float scale, int causal,
                  int window, cudaStream_t st, const uint8_t* bmask = nullptr, long long bmask_hs = 0,
                  const int* seqlens = nullptr) {
  fa::SimtParams s = simt_params(B, H, Hkv, N, scale, causal, window);
  s.bmask = bmask;
  s.bmask_hs = bmask_hs;
  s.nbt = (N + 127) / 128;
  s.seqlens = seqlens;
  s.q = static_cast<const float*>(q);
  s.k = static_cast<const float*>(k);
  s.v = static_cast<const float*>(v);
  s.o = static_cast<const float*>(o);
  s.dout = static_cast<const float*>(dout);
  s.lse = lse;
  s.dq = static_cast<float*>(dq);
  s.dk = static_cast<float*>(dk);
  s.dv = static_cast<float*>(dv);
  s.Drow = static_cast<float*>(ws);
  const size_t rows = static_cast<size_t>(B) * H * N;
  fa::bwd_rowdot_f32_kernel<D><<<static_cast<unsigned>((rows + fa::kSimtRows - 1) / fa::kSimtRows),
                                 32 * fa::kSimtRows, 0, st>>>(s);
  if (launched() != FA_OK) return FA_ERR_CUDA;
  dim3 gkv((N + fa::kSimtRows - 1) / fa::kSimtRows, B * Hkv);
  mark_start(st);
  fa::bwd_dkdv_f32_kernel<D><<<gkv, 32 * fa::kSimtRows, 0, st>>>(s);
  mark_stop(st);
  if (launched() != FA_OK) return FA_ERR_CUDA;
  dim3 gq((N + fa::kSimtRows - 1) / fa::kSimtRows, B * H);
  fa::bwd_dq_f32_kernel<D><<<gq, 32 * fa::kSimtRows, 0, st>>>(s);
  return launched();
}

}  // namespace

extern "C" {

int fa_version(void) { return kAbiVersion; }

void fa_set_timing_events(void* start, void* stop) {
  g_ev_start = static_cast<cudaEvent_t>(start);
  g_ev_stop = static_cast<cudaEvent_t>(stop);
}

const char* fa_status_string(fa_status s) {
  switch (s) {
    case FA_OK: return "ok";
    case FA_ERR_INVALID_ARG: return "invalid argument";
    case FA_ERR_UNSUPPORTED: return "unsupported configuration";
    case FA_ERR_MISALIGNED: return "pointer not 16-byte aligned";
    case FA_ERR_WORKSPACE: return "workspace missing or too small";
    case FA_ERR_CUDA: return "CUDA error";
    case FA_ERR_TIMEOUT: return "device-side wait timed out";
  }
  return "unknown status";
}

fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Hkv, int N,
                 int d, float scale, int causal, int window, fa_dtype dtype, void* stream) {
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
  fa_status s = check_common(B, H, Hkv, N, d, scale, window, dtype);
  if (s != FA_OK) return s;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse)) return FA_ERR_MISALIGNED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == FA_BF16)
    return d == 64 ? fwd_bf16<64>(q, k, v, o, lse, B, H, Hkv, N, scale, causal, window, st)
                   : fwd_bf16<128>(q, k, v, o, lse, B, H, Hkv, N, scale, causal, window, st);
  return d == 64 ? fwd_f32<64>(q, k, v, o, lse, B, H, Hkv, N, scale, causal, window, st)
                 : fwd_f32<128>(q, k, v, o, lse, B, H, Hkv, N, scale, causal, window, st);
}

size_t fa_fwd_splitkv_workspace_size(int B, int H, int N, int d, int num_splits) {
  if (check_common(B, H, 1, N, d, 1.0f, -1, FA_BF16) != FA_OK) return 0;
  if (num_splits < 1 || num_splits > fa::kMaxSplits) return 0;
  return splitkv_ws_bytes(B, H, N, d, num_splits);
}

fa_status fa_fwd_splitkv(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Hkv,
                         int N, int d, float scale, int causal, int window, int num_splits, void* workspace,
                         size_t ws_bytes, fa_dtype dtype, void* stream) {
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
  fa_status s = check_common(B, H, Hkv, N, d, scale, window, dtype);
  if (s != FA_OK) return s;
  if (num_splits < 1 || num_splits > fa::kMaxSplits) return FA_ERR_INVALID_ARG;
  if (dtype != FA_BF16) return FA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse)) return FA_ERR_MISALIGNED;
  if (!workspace || ws_bytes < splitkv_ws_bytes(B, H, N, d, num_splits)) return FA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return FA_ERR_MISALIGNED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return d == 64 ? fwd_bf16<64>(q, k, v, o, lse, B, H, Hkv, N, scale, causal, window, st, num_splits, workspace)
                 : fwd_bf16<128>(q, k, v, o, lse, B, H, Hkv, N, scale, causal, window, st, num_splits, workspace);
}

fa_status fa_fwd_blocksparse(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                             int Hkv, int N, int d, float scale, int causal, int window, const unsigned char* block_mask,
                             long long mask_head_stride, fa_dtype dtype, void* stream) {
  if (!q || !k || !v || !o || !lse || !block_mask) return FA_ERR_INVALID_ARG;
  fa_status s = check_common(B, H, Hkv, N, d, scale, window, dtype);
  if (s != FA_OK) return s;
  if (mask_head_stride < 0) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse)) return FA_ERR_MISALIGNED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == FA_BF16)
    return d == 64 ? fwd_bf16<64>(q, k, v, o, lse, B, H, Hkv, N, scale, causal, window, st, 0, nullptr, block_mask,
                                  mask_head_stride)
                   : fwd_bf16<128>(q, k, v, o, lse, B, H, Hkv, N, scale, causal, window, st, 0, nullptr, block_mask,
                                   mask_head_stride);
  return d == 64 ? fwd_f32<64>(q, k, v, o, lse, B, H, Hkv, N, scale, causal, window, st, block_mask, mask_head_stride)
                 : fwd_f32<128>(q, k, v, o, lse, B, H, Hkv, N, scale, causal, window, st, block_mask, mask_head_stride);
}

fa_status fa_bwd_blocksparse(const void* q, const void* k, const void* v, const void* o, const void* dout,
                             const float* lse, void* dq, void* dk, void* dv, void* workspace, size_t ws_bytes, int B,
                             int H, int Hkv, int N, int d, float scale, int causal, int window,
                             const unsigned char* block_mask, long long mask_head_stride, fa_dtype dtype,
                             void* stream) {
  if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv || !block_mask) return FA_ERR_INVALID_ARG;
  fa_status s = check_common(B, H, Hkv, N, d, scale, window, dtype);
  if (s != FA_OK) return s;
  if (mask_head_stride < 0) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) || !aligned16(lse) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return FA_ERR_MISALIGNED;
  if (!workspace || ws_bytes < ws_layout(B, H, N, d, dtype).total) return FA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return FA_ERR_MISALIGNED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const long long hs = mask_head_stride;
  if (dtype == FA_BF16)
    return d == 64 ? bwd_bf16<64>(q, k, v, o, dout, lse, dq, dk, dv, workspace, B, H, Hkv, N, scale, causal, window, st,
                                  block_mask, hs)
                   : bwd_bf16<128>(q, k, v, o, dout, lse, dq, dk, dv, workspace, B, H, Hkv, N, scale, causal, window,
                                   st, block_mask, hs);
  return d == 64 ? bwd_f32<64>(q, k, v, o, dout, lse, dq, dk, dv, workspace, B, H, Hkv, N, scale, causal, window, st,
                               block_mask, hs)
                 : bwd_f32<128>(q, k, v, o, dout, lse, dq, dk, dv, workspace, B, H, Hkv, N, scale, causal, window, st,
                                block_mask, hs);
}

fa_status fa_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Hkv,
                        int N, int d, float scale, int causal, int window, const int* seqlens, fa_dtype dtype,
                        void* stream) {
  if (!q || !k || !v || !o || !lse || !seqlens) return FA_ERR_INVALID_ARG;
  fa_status s = check_common(B, H, Hkv, N, d, scale, window, dtype);
  if (s != FA_OK) return s;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse)) return FA_ERR_MISALIGNED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == FA_BF16)
    return d == 64 ? fwd_bf16<64>(q, k, v, o, lse, B, H, Hkv, N, scale, causal, window, st, 0, nullptr, nullptr, 0,
                                  seqlens)
                   : fwd_bf16<128>(q, k, v, o, lse, B, H, Hkv, N, scale, causal, window, st, 0, nullptr, nullptr, 0,
                                   seqlens);
  return d == 64 ? fwd_f32<64>(q, k, v, o, lse, B, H, Hkv, N, scale, causal, window, st, nullptr, 0, seqlens)
                 : fwd_f32<128>(q, k, v, o, lse, B, H, Hkv, N, scale, causal, window, st, nullptr, 0, seqlens);
}

fa_status fa_bwd_varlen(const void* q, const void* k, const void* v, const void* o, const void* dout,
                        const float* lse, void* dq, void* dk, void* dv, void* workspace, size_t ws_bytes, int B, int H,
                        int Hkv, int N, int d, float scale, int causal, int window, const int* seqlens,
                        fa_dtype dtype, void* stream) {
  if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv || !seqlens) return FA_ERR_INVALID_ARG;
  fa_status s = check_common(B, H, Hkv, N, d, scale, window, dtype);
  if (s != FA_OK) return s;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) || !aligned16(lse) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return FA_ERR_MISALIGNED;
  if (!workspace || ws_bytes < ws_layout(B, H, N, d, dtype).total) return FA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return FA_ERR_MISALIGNED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == FA_BF16)
    return d == 64 ? bwd_bf16<64>(q, k, v, o, dout, lse, dq, dk, dv, workspace, B, H, Hkv, N, scale, causal, window, st,
                                  nullptr, 0, seqlens)
                   : bwd_bf16<128>(q, k, v, o, dout, lse, dq, dk, dv, workspace, B, H, Hkv, N, scale, causal, window,
                                   st, nullptr, 0, seqlens);
  return d == 64 ? bwd_f32<64>(q, k, v, o, dout, lse, dq, dk, dv, workspace, B, H, Hkv, N, scale, causal, window, st,
                               nullptr, 0, seqlens)
                 : bwd_f32<128>(q, k, v, o, dout, lse, dq, dk, dv, workspace, B, H, Hkv, N, scale, causal, window, st,
                                nullptr, 0, seqlens);
}

size_t fa_bwd_workspace_size(int B, int H, int N, int d, fa_dtype dtype) {
  if (check_common(B, H, 1, N, d, 1.0f, -1, dtype) != FA_OK) return 0;
  return ws_layout(B, H, N, d, dtype).total;
}

fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
                 void* dq, void* dk, void* dv, void* workspace, size_t ws_bytes, int B, int H, int Hkv, int N, int d,
                 float scale, int causal, int window, fa_dtype dtype, void* stream) {
  if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv) return FA_ERR_INVALID_ARG;
  fa_status s = check_common(B, H, Hkv, N, d, scale, window, dtype);
  if (s != FA_OK) return s;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) || !aligned16(lse) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return FA_ERR_MISALIGNED;
  if (!workspace || ws_bytes < ws_layout(B, H, N, d, dtype).total) return FA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return FA_ERR_MISALIGNED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == FA_BF16)
    return d == 64 ? bwd_bf16<64>(q, k, v, o, dout, lse, dq, dk, dv, workspace, B, H, Hkv, N, scale, causal, window, st)
                   : bwd_bf16<128>(q, k, v, o, dout, lse, dq, dk, dv, workspace, B, H, Hkv, N, scale, causal, window,
                                   st);
  return d == 64 ? bwd_f32<64>(q, k, v, o, dout, lse, dq, dk, dv, workspace, B, H, Hkv, N, scale, causal, window, st)
                 : bwd_f32<128>(q, k, v, o, dout, lse, dq, dk, dv, workspace, B, H, Hkv, N, scale, causal, window, st);
}

fa_status fa_last_device_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return FA_ERR_CUDA;
  unsigned int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, fa::g_status, sizeof(v)) != cudaSuccess) return FA_ERR_CUDA;
  if (v != 0 && cudaMemcpyToSymbol(fa::g_status, &zero, sizeof(zero)) != cudaSuccess) return FA_ERR_CUDA;
  if (v & fa::kStatusTimeout) return FA_ERR_TIMEOUT;
  return v ? FA_ERR_CUDA : FA_OK;
}

}  // extern "C"

// ---------------------------------------------------------------- fa_bwd_noalloc
// Scratch for callers that cannot allocate: one file-scope device array per GPU
// that loads this library.  Host code must not pass `g_bwd_scratch` itself to a
// kernel (in host code it names a host-side shadow); its device address comes
// from cudaGetSymbolAddress, looked up once per device and cached.
namespace {

static __device__ __align__(256) unsigned char g_bwd_scratch[FA_BWD_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;

fa_status noalloc_scratch(void** out) {
  static std::mutex mu;
  static void* addr[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_bwd_scratch) != cudaSuccess || p == nullptr) return FA_ERR_CUDA;
    addr[dev] = p;
  }
  *out = addr[dev];
  return FA_OK;
}

}  // namespace

extern "C" fa_status fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const void* dout,
                                    const float* lse, void* dq, void* dk, void* dv, int B, int H, int Hkv, int N,
                                    int d, float scale, int causal, int window, fa_dtype dtype, void* stream) {
  if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv) return FA_ERR_INVALID_ARG;
  fa_status s = check_common(B, H, Hkv, N, d, scale, window, dtype);
  if (s != FA_OK) return s;
  if (ws_layout(B, H, N, d, dtype).total > FA_BWD_NOALLOC_SCRATCH_BYTES) return FA_ERR_WORKSPACE;
  void* scratch = nullptr;
  s = noalloc_scratch(&scratch);
  if (s != FA_OK) return s;
  return fa_bwd(q, k, v, o, dout, lse, dq, dk, dv, scratch, FA_BWD_NOALLOC_SCRATCH_BYTES, B, H, Hkv, N, d, scale,
                causal, window, dtype, stream);
}
