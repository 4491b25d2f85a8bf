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
#include "fwd_persist_sm100.cuh"
#include "fwd_sm100.cuh"
#include "simt_f32.cuh"

namespace {

constexpr int kAbiVersion = 101;

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

// A [B, heads, N, d] bf16 tensor (d contiguous, other axes at the given element
// strides) in 128-row x 64-column boxes with the 128-byte swizzle (the layout
// the UMMA descriptors expect).  When the batch axis steps exactly over all
// heads (every contiguous layout, and slices of longer buffers) the two axes
// merge and the map is 3-D (d, N, B * heads): the TMA unit serves those boxes
// measurably faster than 4-D ones.  Otherwise (e.g. [B, N, H, d]) it is 4-D
// (d, N, heads, B); *four reports which.  Rows past N are zero-filled on load
// and clipped on store, so a tile never reaches another head's or batch
// entry's rows whatever the strides.
bool encode_tile_map(CUtensorMap* m, const void* ptr, int B, int heads, int N, int d, const fa::Strides& s,
                     bool* four) {
  EncodeTiledFn enc = get_encode();
  if (!enc) return false;
  *four = !(B == 1 || s.b == static_cast<long long>(heads) * s.h);
  const int rank = *four ? 4 : 3;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                        static_cast<cuuint64_t>(*four ? heads : static_cast<long long>(B) * heads),
                        static_cast<cuuint64_t>(B)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(s.n) * 2, static_cast<cuuint64_t>(s.h) * 2,
                           static_cast<cuuint64_t>(s.b) * 2};
  cuuint32_t box[4] = {64, 128, 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(ptr), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Encoded maps are cached by everything they encode (address, sizes, strides):
// a hit is exactly the map a fresh encode would give, so the cache needs no
// invalidation when buffers are freed and reused.  A small ring, shared by all
// threads under a mutex.
struct TileMapKey {
  const void* ptr;
  int B, heads, N, d;
  long long sb, sh, sn;
  bool operator==(const TileMapKey& o) const {
    return ptr == o.ptr && B == o.B && heads == o.heads && N == o.N && d == o.d && sb == o.sb && sh == o.sh &&
           sn == o.sn;
  }
};
struct TileMapEntry {
  TileMapKey key;
  CUtensorMap map;
  bool four;
  bool used;
};
constexpr int kTileMapCache = 64;

bool make_tile_map(CUtensorMap* m, const void* ptr, int B, int heads, int N, int d, const fa::Strides& s,
                   bool* four) {
  static std::mutex mu;
  static TileMapEntry cache[kTileMapCache];
  static int next = 0;
  const TileMapKey key{ptr, B, heads, N, d, s.b, s.h, s.n};
  {
    std::lock_guard<std::mutex> lock(mu);
    for (const TileMapEntry& e : cache)
      if (e.used && e.key == key) {
        *m = e.map;
        *four = e.four;
        return true;
      }
  }
  if (!encode_tile_map(m, ptr, B, heads, N, d, s, four)) return false;
  std::lock_guard<std::mutex> lock(mu);
  cache[next] = TileMapEntry{key, *m, *four, true};
  next = (next + 1) % kTileMapCache;
  return true;
}

// Element strides of every tensor argument of one call.
struct Layouts {
  fa::Strides q, k, v, o, dout, dq, dk, dv;
};

// Packed variable lengths in one launch: the B sequences' offsets (device
// copy, read by the kernels) and the total row count T of the packed tensors.
struct Packed {
  const int* rowoff;
  int T;
};

Layouts contiguous_layouts(int B, int H, int Hkv, int N, int d) {
  (void)B;
  const fa::Strides qs = fa::contiguous_strides(H, N, d), ks = fa::contiguous_strides(Hkv, N, d);
  return Layouts{qs, ks, ks, qs, qs, qs, ks, ks};
}

// True when the first n layouts (in q, k, v, o, dout, dq, dk, dv order) equal
// those of b: such calls take the plain (contiguous) kernels.
bool same_layouts(const Layouts& a, const Layouts& b, int n) {
  const fa::Strides* x[8] = {&a.q, &a.k, &a.v, &a.o, &a.dout, &a.dq, &a.dk, &a.dv};
  const fa::Strides* y[8] = {&b.q, &b.k, &b.v, &b.o, &b.dout, &b.dq, &b.dk, &b.dv};
  for (int t = 0; t < n; ++t)
    if (x[t]->b != y[t]->b || x[t]->h != y[t]->h || x[t]->n != y[t]->n) return false;
  return true;
}

// Caller-supplied strides.  Every stride must be positive, a multiple of 16
// bytes and below 2^40 bytes (the tensor-map limits); an axis of extent 1 has
// its stride replaced by the row stride (it is never stepped).  Output layouts
// must be one-to-one: sorted by stride, each axis must step past the whole
// extent of the axes inside it, so that no two output elements share an address.
fa_status check_strides(const fa::Strides& s, int B, int heads, int N, int d, int esize, bool output,
                        fa::Strides* out) {
  fa::Strides t = s;
  if (t.n <= 0) return FA_ERR_INVALID_ARG;
  if (B == 1) t.b = t.n;
  if (heads == 1) t.h = t.n;
  const long long lim = (1LL << 40) / esize;
  for (long long x : {t.b, t.h, t.n}) {
    if (x <= 0 || x >= lim) return FA_ERR_INVALID_ARG;
    if ((x * esize) % 16 != 0) return FA_ERR_MISALIGNED;
  }
  if (output) {
    struct Axis {
      long long stride, extent;
    } ax[3] = {{t.n, N}, {t.h, heads}, {t.b, B}};
    std::sort(ax, ax + 3, [](const Axis& a, const Axis& b) { return a.stride < b.stride; });
    long long span = d;  // elements covered by the axes already placed
    for (const Axis& a : ax) {
      if (a.extent == 1) continue;
      if (a.stride < span) return FA_ERR_INVALID_ARG;
      span = a.stride * a.extent;
    }
  }
  *out = t;
  return FA_OK;
}

// Streaming multiprocessors of the current device (queried once per device);
// 0 if the query fails.
int sm_count() {
  static std::mutex mu;
  static int count[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  std::lock_guard<std::mutex> lock(mu);
  if (count[dev] == 0 && cudaDeviceGetAttribute(&count[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    count[dev] = 0;
  return count[dev];
}

// Raises a kernel's dynamic shared-memory limit, once per (kernel, device):
// the raised limits are remembered by kernel address and device.
template <typename K>
bool set_smem(K kernel, int bytes) {
  struct Done {
    const void* fn;
    int dev, bytes;
  };
  static std::mutex mu;
  static Done done[256];
  static int ndone = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  const void* fn = reinterpret_cast<const void*>(kernel);
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < ndone; ++i)
    if (done[i].fn == fn && done[i].dev == dev && done[i].bytes == bytes) return true;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess) return false;
  if (ndone < 256) done[ndone++] = Done{fn, dev, bytes};
  return true;
}

// Launches one kernel and reports that launch's own outcome (an error left
// behind by an earlier, unrelated call is not taken for this one).
template <typename... KArgs, typename... Args>
fa_status launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...) == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

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

// Decode partials: the g query heads of a kv head form one virtual head of
// g * Nq rows.
inline size_t decode_ws_bytes(int B, int H, int Hkv, int Nq, int d, int splits) {
  return splitkv_ws_bytes(B, Hkv, (H / Hkv) * Nq, d, splits);
}

// splits == 0: the plain forward; splits >= 1: split-KV partials into `ws`
// followed by the merge kernel.  L: non-null for a layout other than the
// contiguous one (then no splits and no block mask); those calls run the
// strided instantiation, the contiguous ones the plain kernels.
template <int D>
fa_status fwd_bf16(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Hkv, int N,
                   float scale, int causal, int window, cudaStream_t st, const Layouts* L = nullptr, int splits = 0,
                   void* ws = nullptr, const uint8_t* bmask = nullptr, long long bmask_hs = 0,
                   const int* seqlens = nullptr, const Packed* pk = nullptr) {
  fa_status ls = FA_OK;
  using C = fa::FwdCfg<D>;
  const Layouts lay = L ? *L : contiguous_layouts(B, H, Hkv, N, D);
  CUtensorMap tq, tk, tv, to;
  bool f4[4];
  // packed: the maps cover all T rows as one batch entry; N is the longest sequence
  const int mB = pk ? 1 : B, mN = pk ? pk->T : N;
  if (!make_tile_map(&tq, q, mB, H, mN, D, lay.q, &f4[0]) || !make_tile_map(&tk, k, mB, Hkv, mN, D, lay.k, &f4[1]) ||
      !make_tile_map(&tv, v, mB, Hkv, mN, D, lay.v, &f4[2]) || !make_tile_map(&to, o, mB, H, mN, D, lay.o, &f4[3]))
    return FA_ERR_CUDA;
  if (!set_smem(fa::fwd_sm100_kernel<D, false, false>, C::kSmemBytes) ||
      !set_smem(fa::fwd_sm100_kernel<D, true, false>, C::kSmemBytes) ||
      !set_smem(fa::fwd_sm100_kernel<D, false, true>, C::kSmemBytes) ||
      !set_smem(fa::fwd_sm100_kernel<D, false, false, true>, C::kSmemBytes) ||
      !set_smem(fa::fwd_persist_kernel<D, false>, fa::FwdPersistCfg<D>::kSmemBytes) ||
      !set_smem(fa::fwd_persist_kernel<D, true>, fa::FwdPersistCfg<D>::kSmemBytes))
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
  // Persistent kernel (at most one CTA per SM, each running units one after
  // another, the next unit's Q load and first products overlapping this one's
  // last tiles and epilogue) when units are short: a unit's fixed cost (CTA
  // start, first loads, epilogue) is then a large share of its time.  Long
  // units keep one CTA each (measured: at 33 key tiles per unit the one-unit
  // kernel is 2-3% faster, at 3 the persistent one 16%).  Block-sparse units
  // differ in work, so there every unit keeps its own CTA and the hardware
  // balances them.
  const int sms = sm_count();
  if (sms <= 0) return FA_ERR_CUDA;
  double tiles_per_unit = causal ? p.npairs + 1.0 : p.ntiles_kv;  // causal pair i: 2i + 2 key tiles
  if (window >= 0) tiles_per_unit = std::min(tiles_per_unit, 2.0 * window / 128.0 + 3.0);
  const bool persist = splits == 0 && !bmask && grid > static_cast<unsigned>(sms) && tiles_per_unit <= 12.0;
  const unsigned pgrid = persist ? static_cast<unsigned>(sms) : grid;
  // Under a causal mask pair i has 2i + 2 key tiles: the persistent CTAs take
  // the units heaviest first across all heads (one group), so each pass over
  // the CTAs holds units of nearly equal work and the passes alternate
  // direction; head groups would restart at the heaviest pairs every group and
  // leave the CTAs unbalanced.
  if (persist && causal) p.group = B * H;
  if (L) {
    if (splits != 0 || bmask) return FA_ERR_UNSUPPORTED;
    fa::FwdStridedParams ps{};
    static_cast<fa::FwdParams&>(ps) = p;
    ps.map4 = (f4[0] ? fa::kMapQ : 0u) | (f4[1] ? fa::kMapK : 0u) | (f4[2] ? fa::kMapV : 0u) |
              (f4[3] ? fa::kMapO : 0u);
    if (pk) {
      ps.rowoff = pk->rowoff;
      ps.T = pk->T;
      ps.o = o;
      ps.o_rs = lay.o.n;
      ps.o_hs = lay.o.h;
    }
    mark_start(st);
    if (persist)
      ls = launch(fa::fwd_persist_kernel<D, true>, pgrid, C::kThreads, fa::FwdPersistCfg<D>::kSmemBytes, st, tq, tk,
                  tv, to, ps);
    else
      ls = launch(fa::fwd_sm100_kernel<D, false, false, true>, grid, C::kThreads, C::kSmemBytes, st, tq, tk, tv, to,
                  ps);
    mark_stop(st);
    return ls;
  }
  if (splits == 0) {
    mark_start(st);
    if (bmask)
      ls = launch(fa::fwd_sm100_kernel<D, false, true>, grid, C::kThreads, C::kSmemBytes, st, tq, tk, tv, to, p);
    else if (persist)
      ls = launch(fa::fwd_persist_kernel<D, false>, pgrid, C::kThreads, fa::FwdPersistCfg<D>::kSmemBytes, st, tq, tk,
                  tv, to, p);
    else
      ls = launch(fa::fwd_sm100_kernel<D, false, false>, grid, C::kThreads, C::kSmemBytes, st, tq, tk, tv, to, p);
    mark_stop(st);
    return ls;
  }
  p.splits = splits;
  p.nq2 = p.npairs * 256;
  p.part_o = static_cast<float*>(ws);
  p.part_m = reinterpret_cast<float4*>(static_cast<uint8_t*>(ws) +
                                       align256(static_cast<size_t>(splits) * B * H * p.nq2 * D * 4));
  mark_start(st);
  ls = launch(fa::fwd_sm100_kernel<D, true, false>, grid * splits, C::kThreads, C::kSmemBytes, st, tq, tk, tv, to, p);
  mark_stop(st);
  if (ls != FA_OK) return ls;
  const unsigned cgrid = static_cast<unsigned>(B * H) * ((N + 31) / 32);
  ls = launch(fa::fwd_combine_kernel<D>, cgrid, 256, 0, st, p, o);
  return ls;
}

// Fewer queries than keys (decode): Nq query rows at positions Nk - Nq + i
// against Nk keys, always through the split-KV kernel and the merge.  The g
// query heads of a kv head are adjacent in [B, H, Nq, d], so they are handed to
// the kernel as one virtual head of g * Nq rows ([B, Hkv, g * Nq, d], the same
// memory; likewise the logsumexp): each CTA then reads a K/V tile once for the
// whole group instead of once per query head.
template <int D>
fa_status fwd_decode_bf16(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Hkv,
                          int Nq, int Nk, float scale, int causal, int window, cudaStream_t st, int splits, void* ws) {
  fa_status ls = FA_OK;
  using C = fa::FwdCfg<D>;
  const int g = H / Hkv, Nv = g * Nq;  // rows of a virtual head
  CUtensorMap tq, tk, tv, to;
  bool f4[4];
  if (!make_tile_map(&tq, q, B, Hkv, Nv, D, fa::contiguous_strides(Hkv, Nv, D), &f4[0]) ||
      !make_tile_map(&tk, k, B, Hkv, Nk, D, fa::contiguous_strides(Hkv, Nk, D), &f4[1]) ||
      !make_tile_map(&tv, v, B, Hkv, Nk, D, fa::contiguous_strides(Hkv, Nk, D), &f4[2]) ||
      !make_tile_map(&to, o, B, Hkv, Nv, D, fa::contiguous_strides(Hkv, Nv, D), &f4[3]))
    return FA_ERR_CUDA;
  if (!set_smem(fa::fwd_sm100_kernel<D, true, false, false, true>, C::kSmemBytes)) return FA_ERR_CUDA;
  fa::FwdDecodeParams p{};
  p.lse = lse;
  p.B = B;
  p.H = Hkv;
  p.Hkv = Hkv;
  p.N = Nv;
  p.g = 1;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.causal = causal ? 1 : 0;
  p.window = window;
  p.npairs = (Nv + 255) / 256;
  p.ntiles_kv = (Nk + 127) / 128;
  p.nbt = p.ntiles_kv;
  p.Nk = Nk;
  p.qoff = Nk - Nq;
  p.nq = Nq;
  {  // virtual heads per group: their Q, O and K, V within ~64 MiB of L2
    const double unit = static_cast<double>(D) * (4.0 * Nv + 4.0 * Nk);
    p.group = std::min(B * Hkv, static_cast<int>(std::max(1.0, std::floor((64.0 * 1024 * 1024) / unit))));
  }
  p.splits = splits;
  p.nq2 = p.npairs * 256;
  p.part_o = static_cast<float*>(ws);
  p.part_m = reinterpret_cast<float4*>(static_cast<uint8_t*>(ws) +
                                       align256(static_cast<size_t>(splits) * B * Hkv * p.nq2 * D * 4));
  const unsigned grid = static_cast<unsigned>(p.npairs) * B * Hkv * splits;
  mark_start(st);
  ls = launch(fa::fwd_sm100_kernel<D, true, false, false, true>, grid, C::kThreads, C::kSmemBytes, st, tq, tk, tv,
              to, p);
  mark_stop(st);
  if (ls != FA_OK) return ls;
  const unsigned cgrid = static_cast<unsigned>(B * Hkv) * ((Nv + 31) / 32);
  ls = launch(fa::fwd_combine_kernel<D>, cgrid, 256, 0, st, static_cast<const fa::FwdParams&>(p), o);
  return ls;
}

void set_simt_strides(fa::SimtParams& s, const Layouts& L) {
  s.sq = L.q;
  s.sk = L.k;
  s.sv = L.v;
  s.so = L.o;
  s.sdo = L.dout;
  s.sdq = L.dq;
  s.sdk = L.dk;
  s.sdv = L.dv;
}

template <int D>
fa_status fwd_f32(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Hkv, int N,
                  float scale, int causal, int window, cudaStream_t st, const Layouts* L = nullptr,
                  const uint8_t* bmask = nullptr, long long bmask_hs = 0, const int* seqlens = nullptr) {
  fa_status ls = FA_OK;
  fa::SimtParams s = simt_params(B, H, Hkv, N, scale, causal, window);
  set_simt_strides(s, L ? *L : contiguous_layouts(B, H, Hkv, N, D));
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
  ls = launch(fa::fwd_simt_f32_kernel<D>, grid, 32 * fa::kSimtRows, 0, st, s);
  mark_stop(st);
  return ls;
}

struct WsLayout {
  size_t nlse2, nd, dqacc, total;
};
// Workspace rows per head of a packed backward: every sequence's rows padded to
// whole 128-row tiles, at 128-aligned starts (packed_ws_row in the kernels).
int packed_ws_rows(int T, int B) { return 128 * ((T + 127) / 128 + B); }
WsLayout ws_layout(int B, int H, int N, int d, fa_dtype dtype) {
  WsLayout w{};
  if (dtype == FA_FP32) {
    w.nd = 0;
    w.total = align256(static_cast<size_t>(B) * H * N * 4);
    return w;
  }
  const size_t rows = static_cast<size_t>(B) * H * padded_rows(N);
  w.nlse2 = 0;
  w.nd = align256(rows * 4);
  w.dqacc = w.nd + align256(rows * 4);
  w.total = w.dqacc + align256(rows * d * 4);
  return w;
}

template <int D>
fa_status bwd_bf16(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
                   void* dq, void* dk, void* dv, void* ws, int B, int H, int Hkv, int N, float scale, int causal,
                   int window, cudaStream_t st, const Layouts* L = nullptr, const uint8_t* bmask = nullptr,
                   long long bmask_hs = 0, const int* seqlens = nullptr, const Packed* pk = nullptr) {
  fa_status ls = FA_OK;
  using C = fa::BwdCfg<D>;
  // packed: each head's workspace rows hold every sequence's padded rows (tp of them)
  const int tp = pk ? packed_ws_rows(pk->T, B) : 0;
  const WsLayout w = pk ? ws_layout(1, H, tp, D, FA_BF16) : ws_layout(B, H, N, D, FA_BF16);
  const Layouts lay = L ? *L : contiguous_layouts(B, H, Hkv, N, D);
  uint8_t* wb = static_cast<uint8_t*>(ws);
  fa::BwdParams p{};
  p.lse = lse;
  p.o = o;
  p.dout = dout;
  p.nlse2 = reinterpret_cast<float*>(wb + w.nlse2);
  p.nD = reinterpret_cast<float*>(wb + w.nd);
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
  p.pairs = (causal && window < 0 && !pk) ? 1 : 0;
  // packed: one slot per (sequence, kv head) holding all its key tiles
  p.slots = pk ? 1 : (p.pairs ? (p.ntiles + 1) / 2 : p.ntiles);
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
  bool f4[6];
  const int mB = pk ? 1 : B, mN = pk ? pk->T : N;  // packed: one batch entry of T rows
  if (!make_tile_map(&tq, q, mB, H, mN, D, lay.q, &f4[0]) || !make_tile_map(&tk, k, mB, Hkv, mN, D, lay.k, &f4[1]) ||
      !make_tile_map(&tv, v, mB, Hkv, mN, D, lay.v, &f4[2]) ||
      !make_tile_map(&tdo, dout, mB, H, mN, D, lay.dout, &f4[3]) ||
      !make_tile_map(&tdk, dk, mB, Hkv, mN, D, lay.dk, &f4[4]) ||
      !make_tile_map(&tdv, dv, mB, Hkv, mN, D, lay.dv, &f4[5]))
    return FA_ERR_CUDA;
  if (!set_smem(fa::bwd_sm100_kernel<D, false>, C::kSmemBytes) ||
      !set_smem(fa::bwd_sm100_kernel<D, true>, C::kSmemBytes) ||
      !set_smem(fa::bwd_sm100_kernel<D, false, true>, C::kSmemBytes))
    return FA_ERR_CUDA;
  const size_t rows = pk ? static_cast<size_t>(H) * tp : static_cast<size_t>(B) * H * p.Np;  // workspace rows
  const unsigned pre_grid = static_cast<unsigned>((rows + 8 * fa::kPreRowsPerWarp - 1) / (8 * fa::kPreRowsPerWarp));
  // Persistent: at most one CTA per SM, each running every gridDim-th slot.
  // Block-sparse slots differ in work, so there every slot keeps its own CTA
  // and the hardware balances them.
  const unsigned nslots = static_cast<unsigned>(p.slots) * B * Hkv;
  const int sms = sm_count();
  if (sms <= 0) return FA_ERR_CUDA;
  const unsigned grid = bmask ? nslots : std::min(nslots, static_cast<unsigned>(sms));
  const unsigned dq_grid = static_cast<unsigned>(rows / 32);
  if (L) {
    if (bmask) return FA_ERR_UNSUPPORTED;
    fa::BwdStridedParams ps{};
    static_cast<fa::BwdParams&>(ps) = p;
    ps.so = lay.o;
    ps.sdo = lay.dout;
    ps.sdq = lay.dq;
    ps.map4 = (f4[0] ? fa::kBMapQ : 0u) | (f4[1] ? fa::kBMapK : 0u) | (f4[2] ? fa::kBMapV : 0u) |
              (f4[3] ? fa::kBMapDO : 0u) | (f4[4] ? fa::kBMapDK : 0u) | (f4[5] ? fa::kBMapDV : 0u);
    if (pk) {
      ps.rowoff = pk->rowoff;
      ps.T = pk->T;
      ps.tp = tp;
      ps.dq_first_store = window < 0 ? 1 : 0;
      ps.dk = dk;
      ps.dv = dv;
      ps.kv_rs = lay.dk.n;
      ps.kv_hs = lay.dk.h;
    }
    ls = launch(fa::bwd_pre_kernel<D, true>, pre_grid, 256, 0, st, ps);
    if (ls != FA_OK) return ls;
    mark_start(st);
    ls = launch(fa::bwd_sm100_kernel<D, false, true>, grid, C::kThreads, C::kSmemBytes, st, tq, tk, tv, tdo, tdk,
                tdv, ps);
    mark_stop(st);
    if (ls != FA_OK) return ls;
    ls = launch(fa::bwd_dq_kernel<D, true>, dq_grid, 256, 0, st, ps);
    return ls;
  }
  ls = launch(fa::bwd_pre_kernel<D>, pre_grid, 256, 0, st, p);
  if (ls != FA_OK) return ls;
  mark_start(st);
  if (bmask)
    ls = launch(fa::bwd_sm100_kernel<D, true>, grid, C::kThreads, C::kSmemBytes, st, tq, tk, tv, tdo, tdk, tdv, p);
  else
    ls = launch(fa::bwd_sm100_kernel<D, false>, grid, C::kThreads, C::kSmemBytes, st, tq, tk, tv, tdo, tdk, tdv, p);
  mark_stop(st);
  if (ls != FA_OK) return ls;
  ls = launch(fa::bwd_dq_kernel<D>, dq_grid, 256, 0, st, p);
  return ls;
}

template <int D>
fa_status bwd_f32(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
                  void* dq, void* dk, void* dv, void* ws, int B, int H, int Hkv, int N, float scale, int causal,
                  int window, cudaStream_t st, const Layouts* L = nullptr, const uint8_t* bmask = nullptr,
                  long long bmask_hs = 0, const int* seqlens = nullptr) {
  fa_status ls = FA_OK;
  fa::SimtParams s = simt_params(B, H, Hkv, N, scale, causal, window);
  set_simt_strides(s, L ? *L : contiguous_layouts(B, H, Hkv, N, D));
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
  ls = launch(fa::bwd_rowdot_f32_kernel<D>, static_cast<unsigned>((rows + fa::kSimtRows - 1) / fa::kSimtRows),
              32 * fa::kSimtRows, 0, st, s);
  if (ls != FA_OK) return ls;
  dim3 gkv((N + fa::kSimtRows - 1) / fa::kSimtRows, B * Hkv);
  mark_start(st);
  ls = launch(fa::bwd_dkdv_f32_kernel<D>, gkv, 32 * fa::kSimtRows, 0, st, s);
  mark_stop(st);
  if (ls != FA_OK) return ls;
  dim3 gq((N + fa::kSimtRows - 1) / fa::kSimtRows, B * H);
  ls = launch(fa::bwd_dq_f32_kernel<D>, gq, 32 * fa::kSimtRows, 0, st, s);
  return ls;
}

// ---------------------------------------------------------------- packed variable lengths
// Sequence b is a one-entry problem of len_b = cu[b+1] - cu[b] rows whose
// tensors start at token row cu[b] of the packed buffers (rows H*d elements
// apart, heads d apart): each runs through the strided path with its own tensor
// maps, so loads stop and stores clip at the sequence end.
fa_status packed_lengths(const int* cu, int B, int* max_len) {
  if (!cu || B < 1 || cu[0] != 0) return FA_ERR_INVALID_ARG;
  int m = 0;
  for (int b = 0; b < B; ++b) {
    if (cu[b + 1] < cu[b]) return FA_ERR_INVALID_ARG;
    m = std::max(m, cu[b + 1] - cu[b]);
  }
  *max_len = m;
  return FA_OK;
}

// Packed tensors of T rows in one launch: the row count and the workspace rows
// must stay within int range (tensor-map coordinates and kernel indices).
fa_status check_packed_rows(int T, int B) {
  if (T < 0 || static_cast<long long>(T) + 128LL * (B + 1) > (1LL << 30)) return FA_ERR_INVALID_ARG;
  return FA_OK;
}

// Layouts of sequence b: q, o, dout, dq [len, H, d]; k, v, dk, dv [len, Hkv, d].
fa_status packed_layouts(int H, int Hkv, int len, int d, int es, Layouts* L) {
  const fa::Strides qs{static_cast<long long>(len) * H * d, d, static_cast<long long>(H) * d};
  const fa::Strides ks{static_cast<long long>(len) * Hkv * d, d, static_cast<long long>(Hkv) * d};
  const fa::Strides in[8] = {qs, ks, ks, qs, qs, qs, ks, ks};
  fa::Strides* out[8] = {&L->q, &L->k, &L->v, &L->o, &L->dout, &L->dq, &L->dk, &L->dv};
  const int heads[8] = {H, Hkv, Hkv, H, H, H, Hkv, Hkv};
  for (int t = 0; t < 8; ++t) {
    const fa_status s = check_strides(in[t], 1, heads[t], len, d, es, t == 3 || t >= 5, out[t]);
    if (s != FA_OK) return s;
  }
  return FA_OK;
}

// The kernels run on the current device, where the tensor maps are built and
// the allocation-free scratch address is looked up: a stream of another device
// is an argument error (the legacy default stream, NULL, is the current
// device's).
fa_status check_stream(void* stream) {
  int cur = 0, sdev = 0;
  if (cudaGetDevice(&cur) != cudaSuccess) return FA_ERR_CUDA;
  if (stream == nullptr) return FA_OK;
  if (cudaStreamGetDevice(static_cast<cudaStream_t>(stream), &sdev) != cudaSuccess) return FA_ERR_INVALID_ARG;
  return sdev == cur ? FA_OK : FA_ERR_INVALID_ARG;
}

// dtype / head-dimension dispatch shared by every entry point (arguments
// already checked).
fa_status run_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Hkv, int N,
                  int d, float scale, int causal, int window, fa_dtype dtype, void* stream, const Layouts* L,
                  int splits = 0, void* ws = nullptr, const uint8_t* bmask = nullptr, long long hs = 0,
                  const int* seqlens = nullptr) {
  const fa_status sc = check_stream(stream);
  if (sc != FA_OK) return sc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == FA_BF16)
    return d == 64 ? fwd_bf16<64>(q, k, v, o, lse, B, H, Hkv, N, scale, causal, window, st, L, splits, ws, bmask, hs,
                                  seqlens)
                   : fwd_bf16<128>(q, k, v, o, lse, B, H, Hkv, N, scale, causal, window, st, L, splits, ws, bmask,
                                   hs, seqlens);
  if (splits != 0) return FA_ERR_UNSUPPORTED;
  return d == 64 ? fwd_f32<64>(q, k, v, o, lse, B, H, Hkv, N, scale, causal, window, st, L, bmask, hs, seqlens)
                 : fwd_f32<128>(q, k, v, o, lse, B, H, Hkv, N, scale, causal, window, st, L, bmask, hs, seqlens);
}

fa_status run_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
                  void* dq, void* dk, void* dv, void* ws, int B, int H, int Hkv, int N, int d, float scale, int causal,
                  int window, fa_dtype dtype, void* stream, const Layouts* L, const uint8_t* bmask = nullptr,
                  long long hs = 0, const int* seqlens = nullptr) {
  const fa_status sc = check_stream(stream);
  if (sc != FA_OK) return sc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == FA_BF16)
    return d == 64 ? bwd_bf16<64>(q, k, v, o, dout, lse, dq, dk, dv, ws, B, H, Hkv, N, scale, causal, window, st, L,
                                  bmask, hs, seqlens)
                   : bwd_bf16<128>(q, k, v, o, dout, lse, dq, dk, dv, ws, B, H, Hkv, N, scale, causal, window, st, L,
                                   bmask, hs, seqlens);
  return d == 64 ? bwd_f32<64>(q, k, v, o, dout, lse, dq, dk, dv, ws, B, H, Hkv, N, scale, causal, window, st, L,
                               bmask, hs, seqlens)
                 : bwd_f32<128>(q, k, v, o, dout, lse, dq, dk, dv, ws, B, H, Hkv, N, scale, causal, window, st, L,
                                bmask, hs, seqlens);
}

fa_status check_bwd_buffers(const void* q, const void* k, const void* v, const void* o, const void* dout,
                            const float* lse, const void* dq, const void* dk, const void* dv, const void* workspace,
                            size_t ws_bytes, int B, int H, int N, int d, fa_dtype dtype) {
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) || !aligned16(lse) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return FA_ERR_MISALIGNED;
  if (!workspace || ws_bytes < ws_layout(B, H, N, d, dtype).total) return FA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return FA_ERR_MISALIGNED;
  return FA_OK;
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
  return run_fwd(q, k, v, o, lse, B, H, Hkv, N, d, scale, causal, window, dtype, stream,
                 nullptr);
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
  return run_fwd(q, k, v, o, lse, B, H, Hkv, N, d, scale, causal, window, dtype, stream,
                 nullptr, num_splits, workspace);
}

fa_status fa_fwd_blocksparse(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                             int Hkv, int N, int d, float scale, int causal, int window, const unsigned char* block_mask,
                             long long mask_head_stride, fa_dtype dtype, void* stream) {
  if (!q || !k || !v || !o || !lse || !block_mask) return FA_ERR_INVALID_ARG;
  fa_status s = check_common(B, H, Hkv, N, d, scale, window, dtype);
  if (s != FA_OK) return s;
  if (mask_head_stride < 0) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse)) return FA_ERR_MISALIGNED;
  return run_fwd(q, k, v, o, lse, B, H, Hkv, N, d, scale, causal, window, dtype, stream,
                 nullptr, 0, nullptr, block_mask, mask_head_stride);
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
  s = check_bwd_buffers(q, k, v, o, dout, lse, dq, dk, dv, workspace, ws_bytes, B, H, N, d, dtype);
  if (s != FA_OK) return s;
  return run_bwd(q, k, v, o, dout, lse, dq, dk, dv, workspace, B, H, Hkv, N, d, scale, causal, window, dtype, stream,
                 nullptr, block_mask, mask_head_stride);
}

fa_status fa_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Hkv,
                        int N, int d, float scale, int causal, int window, const int* seqlens, fa_dtype dtype,
                        void* stream) {
  if (!q || !k || !v || !o || !lse || !seqlens) return FA_ERR_INVALID_ARG;
  fa_status s = check_common(B, H, Hkv, N, d, scale, window, dtype);
  if (s != FA_OK) return s;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse)) return FA_ERR_MISALIGNED;
  return run_fwd(q, k, v, o, lse, B, H, Hkv, N, d, scale, causal, window, dtype, stream,
                 nullptr, 0, nullptr, nullptr, 0, seqlens);
}

fa_status fa_bwd_varlen(const void* q, const void* k, const void* v, const void* o, const void* dout,
                        const float* lse, void* dq, void* dk, void* dv, void* workspace, size_t ws_bytes, int B, int H,
                        int Hkv, int N, int d, float scale, int causal, int window, const int* seqlens,
                        fa_dtype dtype, void* stream) {
  if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv || !seqlens) return FA_ERR_INVALID_ARG;
  fa_status s = check_common(B, H, Hkv, N, d, scale, window, dtype);
  if (s != FA_OK) return s;
  s = check_bwd_buffers(q, k, v, o, dout, lse, dq, dk, dv, workspace, ws_bytes, B, H, N, d, dtype);
  if (s != FA_OK) return s;
  return run_bwd(q, k, v, o, dout, lse, dq, dk, dv, workspace, B, H, Hkv, N, d, scale, causal, window, dtype, stream,
                 nullptr, nullptr, 0, seqlens);
}

fa_status fa_fwd_strided(const void* q, const void* k, const void* v, void* o, float* lse, const fa_strides* strides,
                         int B, int H, int Hkv, int N, int d, float scale, int causal, int window, const int* seqlens,
                         fa_dtype dtype, void* stream) {
  if (!q || !k || !v || !o || !lse || !strides) return FA_ERR_INVALID_ARG;
  fa_status s = check_common(B, H, Hkv, N, d, scale, window, dtype);
  if (s != FA_OK) return s;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse)) return FA_ERR_MISALIGNED;
  Layouts L = contiguous_layouts(B, H, Hkv, N, d);
  const int es = dtype == FA_BF16 ? 2 : 4;
  fa::Strides* dst[4] = {&L.q, &L.k, &L.v, &L.o};
  const int heads[4] = {H, Hkv, Hkv, H};
  for (int t = 0; t < 4; ++t) {
    const fa::Strides in{strides[t].batch, strides[t].head, strides[t].row};
    s = check_strides(in, B, heads[t], N, d, es, t == 3, dst[t]);
    if (s != FA_OK) return s;
  }
  const Layouts C0 = contiguous_layouts(B, H, Hkv, N, d);
  const bool contig = same_layouts(L, C0, 4);
  return run_fwd(q, k, v, o, lse, B, H, Hkv, N, d, scale, causal, window, dtype, stream, contig ? nullptr : &L, 0,
                 nullptr, nullptr, 0,
                 seqlens);
}

fa_status fa_bwd_strided(const void* q, const void* k, const void* v, const void* o, const void* dout,
                         const float* lse, void* dq, void* dk, void* dv, const fa_strides* strides, void* workspace,
                         size_t ws_bytes, int B, int H, int Hkv, int N, int d, float scale, int causal, int window,
                         const int* seqlens, fa_dtype dtype, void* stream) {
  if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv || !strides) return FA_ERR_INVALID_ARG;
  fa_status s = check_common(B, H, Hkv, N, d, scale, window, dtype);
  if (s != FA_OK) return s;
  s = check_bwd_buffers(q, k, v, o, dout, lse, dq, dk, dv, workspace, ws_bytes, B, H, N, d, dtype);
  if (s != FA_OK) return s;
  Layouts L = contiguous_layouts(B, H, Hkv, N, d);
  const int es = dtype == FA_BF16 ? 2 : 4;
  fa::Strides* dst[8] = {&L.q, &L.k, &L.v, &L.o, &L.dout, &L.dq, &L.dk, &L.dv};
  const int heads[8] = {H, Hkv, Hkv, H, H, H, Hkv, Hkv};
  for (int t = 0; t < 8; ++t) {
    const fa::Strides in{strides[t].batch, strides[t].head, strides[t].row};
    s = check_strides(in, B, heads[t], N, d, es, t >= 5, dst[t]);
    if (s != FA_OK) return s;
  }
  const Layouts C0 = contiguous_layouts(B, H, Hkv, N, d);
  const bool contig = same_layouts(L, C0, 8);
  return run_bwd(q, k, v, o, dout, lse, dq, dk, dv, workspace, B, H, Hkv, N, d, scale, causal, window, dtype, stream,
                 contig ? nullptr : &L, nullptr, 0, seqlens);
}

size_t fa_fwd_decode_workspace_size(int B, int H, int Hkv, int Nq, int d, int num_splits) {
  if (Nq < 1 || check_common(B, H, Hkv, Nq, d, 1.0f, -1, FA_BF16) != FA_OK) return 0;
  if (num_splits < 1 || num_splits > fa::kMaxSplits) return 0;
  return decode_ws_bytes(B, H, Hkv, Nq, d, num_splits);
}

fa_status fa_fwd_decode(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Hkv,
                        int Nq, int Nk, int d, float scale, int causal, int window, int num_splits, void* workspace,
                        size_t ws_bytes, fa_dtype dtype, void* stream) {
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
  if (Nq < 1 || Nk < Nq) return FA_ERR_INVALID_ARG;
  fa_status s = check_common(B, H, Hkv, Nk, d, scale, window, dtype);
  if (s != FA_OK) return s;
  if (num_splits < 1 || num_splits > fa::kMaxSplits) return FA_ERR_INVALID_ARG;
  if (dtype != FA_BF16) return FA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse)) return FA_ERR_MISALIGNED;
  if (!workspace || ws_bytes < decode_ws_bytes(B, H, Hkv, Nq, d, num_splits)) return FA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return FA_ERR_MISALIGNED;
  if ((s = check_stream(stream)) != FA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return d == 64 ? fwd_decode_bf16<64>(q, k, v, o, lse, B, H, Hkv, Nq, Nk, scale, causal, window, st, num_splits,
                                       workspace)
                 : fwd_decode_bf16<128>(q, k, v, o, lse, B, H, Hkv, Nq, Nk, scale, causal, window, st, num_splits,
                                        workspace);
}

fa_status fa_fwd_packed(const void* q, const void* k, const void* v, void* o, float* lse, const int* cu_seqlens,
                        const int* cu_seqlens_dev, int B, int H, int Hkv, int d, float scale, int causal, int window,
                        fa_dtype dtype, void* stream) {
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
  int max_len = 0;
  fa_status s = packed_lengths(cu_seqlens, B, &max_len);
  if (s != FA_OK) return s;
  s = check_common(1, H, Hkv, std::max(max_len, 1), d, scale, window, dtype);
  if (s != FA_OK) return s;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse)) return FA_ERR_MISALIGNED;
  const size_t es = dtype == FA_BF16 ? 2 : 4;
  const int T = cu_seqlens[B];
  if (T == 0) return FA_OK;
  if (dtype == FA_BF16) {  // one launch over every sequence
    if (!cu_seqlens_dev || !aligned16(cu_seqlens_dev)) return FA_ERR_INVALID_ARG;
    if ((s = check_packed_rows(T, B)) != FA_OK) return s;
    Layouts L{};
    if ((s = packed_layouts(H, Hkv, T, d, static_cast<int>(es), &L)) != FA_OK) return s;
    if ((s = check_stream(stream)) != FA_OK) return s;
    const Packed pk{cu_seqlens_dev, T};
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    return d == 64 ? fwd_bf16<64>(q, k, v, o, lse, B, H, Hkv, max_len, scale, causal, window, st, &L, 0, nullptr,
                                  nullptr, 0, nullptr, &pk)
                   : fwd_bf16<128>(q, k, v, o, lse, B, H, Hkv, max_len, scale, causal, window, st, &L, 0, nullptr,
                                   nullptr, 0, nullptr, &pk);
  }
  for (int b = 0; b < B; ++b) {  // fp32: one launch per sequence
    const int len = cu_seqlens[b + 1] - cu_seqlens[b];
    if (len == 0) continue;
    Layouts L{};
    if ((s = packed_layouts(H, Hkv, len, d, static_cast<int>(es), &L)) != FA_OK) return s;
    const size_t row = static_cast<size_t>(cu_seqlens[b]);
    const size_t oq = row * H * d * es, ok = row * Hkv * d * es;
    s = run_fwd(static_cast<const uint8_t*>(q) + oq, static_cast<const uint8_t*>(k) + ok,
                static_cast<const uint8_t*>(v) + ok, static_cast<uint8_t*>(o) + oq, lse + row * H, 1, H, Hkv, len, d,
                scale, causal, window, dtype, stream, H == 1 && Hkv == 1 ? nullptr : &L);
    if (s != FA_OK) return s;
  }
  return FA_OK;
}

size_t fa_bwd_packed_workspace_size(const int* cu_seqlens, int B, int H, int d, fa_dtype dtype) {
  int max_len = 0;
  if (packed_lengths(cu_seqlens, B, &max_len) != FA_OK) return 0;
  if (check_common(1, H, 1, std::max(max_len, 1), d, 1.0f, -1, dtype) != FA_OK) return 0;
  if (dtype == FA_BF16) {
    if (check_packed_rows(cu_seqlens[B], B) != FA_OK) return 0;
    return ws_layout(1, H, packed_ws_rows(cu_seqlens[B], B), d, dtype).total;
  }
  return ws_layout(1, H, std::max(max_len, 1), d, dtype).total;
}

fa_status fa_bwd_packed(const void* q, const void* k, const void* v, const void* o, const void* dout,
                        const float* lse, void* dq, void* dk, void* dv, const int* cu_seqlens,
                        const int* cu_seqlens_dev, void* workspace, size_t ws_bytes, int B, int H, int Hkv, int d,
                        float scale, int causal, int window, fa_dtype dtype, void* stream) {
  if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv) return FA_ERR_INVALID_ARG;
  int max_len = 0;
  fa_status s = packed_lengths(cu_seqlens, B, &max_len);
  if (s != FA_OK) return s;
  s = check_common(1, H, Hkv, std::max(max_len, 1), d, scale, window, dtype);
  if (s != FA_OK) return s;
  const size_t need = fa_bwd_packed_workspace_size(cu_seqlens, B, H, d, dtype);
  if (need == 0) return FA_ERR_INVALID_ARG;
  s = check_bwd_buffers(q, k, v, o, dout, lse, dq, dk, dv, workspace, ws_bytes, 1, H, std::max(max_len, 1), d,
                        dtype);
  if (s != FA_OK) return s;
  if (ws_bytes < need) return FA_ERR_WORKSPACE;
  const size_t es = dtype == FA_BF16 ? 2 : 4;
  const int T = cu_seqlens[B];
  if (T == 0) return FA_OK;
  if (dtype == FA_BF16) {  // one launch of each backward kernel over every sequence
    if (!cu_seqlens_dev || !aligned16(cu_seqlens_dev)) return FA_ERR_INVALID_ARG;
    Layouts L{};
    if ((s = packed_layouts(H, Hkv, T, d, static_cast<int>(es), &L)) != FA_OK) return s;
    if ((s = check_stream(stream)) != FA_OK) return s;
    const Packed pk{cu_seqlens_dev, T};
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    return d == 64 ? bwd_bf16<64>(q, k, v, o, dout, lse, dq, dk, dv, workspace, B, H, Hkv, max_len, scale, causal,
                                  window, st, &L, nullptr, 0, nullptr, &pk)
                   : bwd_bf16<128>(q, k, v, o, dout, lse, dq, dk, dv, workspace, B, H, Hkv, max_len, scale, causal,
                                   window, st, &L, nullptr, 0, nullptr, &pk);
  }
  for (int b = 0; b < B; ++b) {  // fp32: in stream order, each sequence reuses the workspace after the previous one
    const int len = cu_seqlens[b + 1] - cu_seqlens[b];
    if (len == 0) continue;
    Layouts L{};
    if ((s = packed_layouts(H, Hkv, len, d, static_cast<int>(es), &L)) != FA_OK) return s;
    const size_t row = static_cast<size_t>(cu_seqlens[b]);
    const size_t oq = row * H * d * es, ok = row * Hkv * d * es;
    s = run_bwd(static_cast<const uint8_t*>(q) + oq, static_cast<const uint8_t*>(k) + ok,
                static_cast<const uint8_t*>(v) + ok, static_cast<const uint8_t*>(o) + oq,
                static_cast<const uint8_t*>(dout) + oq, lse + row * H, static_cast<uint8_t*>(dq) + oq,
                static_cast<uint8_t*>(dk) + ok, static_cast<uint8_t*>(dv) + ok, workspace, 1, H, Hkv, len, d, scale,
                causal, window, dtype, stream, H == 1 && Hkv == 1 ? nullptr : &L);
    if (s != FA_OK) return s;
  }
  return FA_OK;
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
  s = check_bwd_buffers(q, k, v, o, dout, lse, dq, dk, dv, workspace, ws_bytes, B, H, N, d, dtype);
  if (s != FA_OK) return s;
  return run_bwd(q, k, v, o, dout, lse, dq, dk, dv, workspace, B, H, Hkv, N, d, scale, causal, window, dtype, stream,
                 nullptr);
}

fa_status fa_debug_set_wait_limit(unsigned long long ns) {
  const unsigned long long v = ns ? ns : fa::kWaitLimitNs;
  return cudaMemcpyToSymbol(fa::g_wait_limit_ns, &v, sizeof(v)) == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status fa_debug_set_stall(int on) {
  const int v = on ? 1 : 0;
  return cudaMemcpyToSymbol(fa::g_debug_stall, &v, sizeof(v)) == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status fa_last_device_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return FA_ERR_CUDA;
  unsigned int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, fa::g_status, sizeof(v)) != cudaSuccess) return FA_ERR_CUDA;
  if (v != 0 && cudaMemcpyToSymbol(fa::g_status, &zero, sizeof(zero)) != cudaSuccess) return FA_ERR_CUDA;
  if (v & fa::kStatusTimeout) return FA_ERR_TIMEOUT;
  return v ? FA_ERR_CUDA : FA_OK;
}

#ifdef FA_TRACE
// Phase-timestamp builds only (not part of the ABI): copies or clears the trace buffer.
constexpr size_t kTraceBytes =
    sizeof(long long) * fa::kTraceCtas * fa::kTraceRoles * fa::kTraceIters * fa::kTraceEvents;
int fa_trace_read(void* dst, size_t bytes) {
  if (bytes > kTraceBytes) bytes = kTraceBytes;
  return cudaMemcpyFromSymbol(dst, fa::g_trace, bytes) == cudaSuccess ? 0 : 1;
}
int fa_trace_cta_read(void* dst, size_t bytes) {
  if (bytes > sizeof(long long) * 16384 * 4) bytes = sizeof(long long) * 16384 * 4;
  return cudaMemcpyFromSymbol(dst, fa::g_trace_cta, bytes) == cudaSuccess ? 0 : 1;
}
int fa_trace_clear(void) {
  static long long zero[kTraceBytes / sizeof(long long)];
  return cudaMemcpyToSymbol(fa::g_trace, zero, sizeof(zero)) == cudaSuccess ? 0 : 1;
}
#endif

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
  if ((s = check_stream(stream)) != FA_OK) return s;  // the scratch address is the current device's
  void* scratch = nullptr;
  s = noalloc_scratch(&scratch);
  if (s != FA_OK) return s;
  return fa_bwd(q, k, v, o, dout, lse, dq, dk, dv, scratch, FA_BWD_NOALLOC_SCRATCH_BYTES, B, H, Hkv, N, d, scale,
                causal, window, dtype, stream);
}
