// bwd_sm100.cuh -- bf16 attention backward on sm_100a tensor cores.
//
// The backward pass recomputes the scores and probabilities tile by tile from
// Q, K and the saved logsumexp instead of reading an N x N matrix ("Flash
// attention and efficient attention", section "Backward Pass: Recomputation";
// "FlashAttention" guide page, "Tiling through SRAM").  The gradient formulas
// are the softmax Jacobian for L = sum(dO * O):
//   dV = P^T dO,  dP = dO V^T,  dS = P * (dP - D),  D_i = dO_i . O_i,
//   dK = scale dS^T Q,  dQ = scale dS K.
//
// Three kernels run on one stream:
//   bwd_pre_kernel   -D_i, -LSE_i * log2(e) (-inf on padding rows) and a
//                    zeroed fp32 dQ accumulator, all in the caller's workspace;
//   bwd_sm100_kernel persistent: each CTA runs a list of jobs, one 128-key tile
//                    of one kv head each: K_j and V_j stay in shared memory
//                    while the CTA walks every query tile (of every query head
//                    of the GQA group) that can see them; dK_j and dV_j
//                    accumulate in TMEM and are written once, dQ partial tiles
//                    are added into the accumulator;
//   bwd_dq_kernel    dQ = bf16(scale * accumulator).
//
// Main-kernel roles (512 threads, four warpgroups):
//   warps 0-3   P / dS for query columns 0-63 of the tile, one thread per key
//               row (TMEM lanes 0-127)
//   warps 4-7   the same for query columns 64-127
//   warps 8-11  dQ drain (one thread per query row of the dQ tile) and each
//               tile's dK/dV epilogue (one thread per key row)
//   warp 12     tcgen05.mma issuer (one thread) and TMEM owner
//   warp 13     TMA producer of the Q tiles and their LSE / D rows
//   warp 14     idle (completes the fourth warpgroup)
//   warp 15     TMA producer of the dO tiles
// Registers: 128 per thread at launch; the fourth warpgroup drops to 96, the
// compute warpgroups rise to 136 and the drain to 144 (136 + 136 + 144 + 96 =
// 4 * 128, checked below; strided instantiations 128 + 128 + 160 + 96), so a
// drain thread holds a whole dQ row and releases the TMEM tile at once.
//
// dQ reduction.  Every (key tile, query tile) pair adds a 128 x D fp32 partial
// into the global accumulator.  The drain loads the partial from TMEM into
// registers (freeing the TMEM tile), writes it to shared memory 32 columns at
// a time and hands each 16 KB chunk to the TMA unit as one bulk reduce-add, so
// the reductions never occupy the load/store queues that the compute warps
// need for their shared-memory traffic.  The accumulator is laid out in the
// same 16 KB chunks (see dqacc_chunk).
//
// The products are formed transposed (S^T = K Q^T, dP^T = V dO^T) so that P^T
// and dS^T land in TMEM with one key row per lane and can be fed back, as
// packed bf16, as the A operand of dV += P^T dO and dK += dS^T Q.  dS itself
// (needed with queries as rows for dQ = dS K) is written to shared memory in
// the MN-major layout the tensor core reads.
// TMEM: S^T [0,128), dP^T [128,256), dV [256,256+D), dK [256+D,256+2D); the dQ
// tile takes [128,256) for D = 128 (after dS^T has been consumed) and
// [384,448) for D = 64.  Each compute warpgroup writes its 64 packed-bf16
// P^T (dS^T) values per row over the first half of its own 64 S^T (dP^T)
// columns, so query column c of the tile lives at packed column
// (c / 64) * 64 + (c % 64) / 2.
#pragma once

#include <type_traits>

#include "sm100_ptx.cuh"

namespace fa {

struct BwdParams {
  const float* lse;  // [B*H*N] from the forward
  const void* o;     // bf16 [B*H*N*D]
  const void* dout;  // bf16 [B*H*N*D]
  float* nlse2;      // workspace [B*H*Np]: -lse*log2(e), -inf on rows >= N
  float* nD;         // workspace [B*H*Np]: -D_i, 0 on rows >= N
  float* dqacc;      // workspace [B*H*Np*D], in 16 KB chunks (dqacc_chunk)
  void* dq;          // bf16 [B*H*N*D]
  int B, H, Hkv, N, Np, g;
  float scale, scale_log2;
  int causal, window;
  int ntiles;  // Np / 128
  int group;   // kv heads per rasterisation group (kept L2-resident together)
  int slots;   // slots (units of work the CTAs take in turn) per kv head
  int pairs;   // 1 (causal): ceil(ntiles / 2) slots, each holding key tiles j and ntiles - 1 - j;
               // 0: ntiles slots of one key tile each (packed: one slot of every key tile)
  // block-sparse mode (non-null bmask): 0/1 per 128 x 128 block, [query block]
  // [key block] per query head, bmask_hs elements apart (0: shared by all heads)
  const uint8_t* bmask;
  long long bmask_hs;
  const int* seqlens;  // padded variable lengths (null: every batch entry has N rows)
};

// Arguments of the strided-layout instantiations: element strides of O and dO
// (read by the preprocess) and of dQ (written by the convert pass), and which
// tensor maps are 4-D (column, row, head, batch entry) rather than 3-D (column,
// row, batch entry * heads + head).  A separate type, so the contiguous
// instantiations keep the plain BwdParams.
struct BwdStridedParams : BwdParams {
  Strides so, sdo, sdq;
  unsigned map4;
  // Packed variable lengths (non-null rowoff, device memory): batch entry b is
  // sequence b, rows rowoff[b] .. rowoff[b+1] - 1 of tensors that hold all T
  // rows back to back (one batch entry in the tensor maps and strides); N is
  // the longest length.  The workspace rows of sequence b start at
  // packed_ws_row(b) inside each head's tp rows; the logsumexp of sequence b is
  // [H, len_b] at lse + rowoff[b] * H; dK and dV rows are stored only up to the
  // sequence end (plain stores for a key tile the end falls inside).
  const int* rowoff;
  int T;
  int tp;  // workspace rows per head: 128 * (ceil(T / 128) + B)
  void* dk;
  void* dv;
  long long kv_rs, kv_hs;  // element strides of dK / dV rows and heads
  // Packed, no window: a sequence's first key tile reaches every one of its
  // query tiles and its job runs first in its slot, so that job stores its dQ
  // partials instead of adding them, and the accumulator needs no zeroing.
  int dq_first_store;
};
// First workspace row of packed sequence b (a multiple of 128): consecutive
// sequences' padded row ranges [start, start + 128 * ceil(len / 128)) never
// overlap, since floor(rowoff[b + 1] / 128) >= floor(rowoff[b] / 128) +
// floor(len_b / 128).
__device__ __forceinline__ int packed_ws_row(int rowoff_b, int b) { return 128 * (rowoff_b / 128 + b); }
// Sequence b's first row and length, clamped to the tensors' T rows.
__device__ __forceinline__ void packed_range(const BwdStridedParams& p, int b, int& rb, int& len) {
  rb = min(max(p.rowoff[b], 0), p.T);
  len = min(min(max(p.rowoff[b + 1], rb), p.T) - rb, p.N);
}
// The packed sequence whose workspace rows hold row R (0 <= R < tp): the last b
// with packed_ws_row(b) <= R (starts increase with b).  Called by a whole warp
// with the same R: each round the 32 lanes probe 32 evenly spaced candidates
// and a ballot narrows the range 32-fold, so 1000 sequences take two rounds of
// loads instead of ten dependent ones.
__device__ __forceinline__ int packed_seq_of_ws_row(const BwdStridedParams& p, int R) {
  const int lane = threadIdx.x & 31;
  int lo = 0, hi = p.B - 1;
  while (lo < hi) {
    const int step = (hi - lo + 32) / 32;  // ceil((hi - lo + 1) / 32)
    const int idx = lo + lane * step;
    const bool le = idx <= hi && packed_ws_row(min(max(p.rowoff[idx], 0), p.T), idx) <= R;
    const int k = __popc(__ballot_sync(0xffffffffu, le));  // probes at or before R: lanes 0 .. k - 1
    if (k == 0) break;  // R before every start (offsets that do not start at 0): sequence lo
    const int nlo = lo + (k - 1) * step;
    hi = min(hi, lo + k * step - 1);
    lo = nlo;
  }
  return lo;
}
constexpr unsigned kBMapQ = 1, kBMapK = 2, kBMapV = 4, kBMapDO = 8, kBMapDK = 16, kBMapDV = 32;
template <bool kStrided>
using BwdArgs = std::conditional_t<kStrided, BwdStridedParams, BwdParams>;

__device__ __forceinline__ int valid_rows(const BwdParams& p, int b) {
  return p.seqlens ? max(0, min(p.seqlens[b], p.N)) : p.N;
}

template <int D>
struct BwdCfg {
  static constexpr int kTileBytes = 128 * D * 2;
  static constexpr int kChunks = D / 64;                 // 64-column chunks of a bf16 tile
  static constexpr int kQStages = (D == 128) ? 2 : 3;    // (Q, LSE, D) tile sets in flight
  static constexpr int kDoStages = (D == 128) ? 1 : 2;   // dO tiles in flight
  // K/V buffers: with two, the next job's K and V load while the current job
  // runs (no room for a second pair at D = 128).
  static constexpr int kKvBufs = (D == 128) ? 1 : 2;
  static constexpr int kDsBytes = 128 * 128 * 2;
  static constexpr int kVecBytes = 2 * 128 * 4;          // -LSE*log2(e) and -D of one query tile
  static constexpr int kDqChunkBytes = 128 * 32 * 4;     // 32 fp32 columns of a 128-row dQ tile
  static constexpr int kDqChunks = D / 32;               // chunks per dQ tile
  static constexpr int kDqStages = 2;                    // staging buffers of the dQ reduction
  static constexpr int kNumBars = 2 * kKvBufs + 2 * kQStages + 2 * kDoStages + 9;
  // The dynamic shared window starts 1024-byte aligned (checked at run time),
  // so no alignment slack is reserved: at D = 128 this is 231,576 of the
  // 232,448 bytes a CTA may use (216,264 at D = 64).
  static constexpr int kSmemBytes = 2 * kKvBufs * kTileBytes + kQStages * kTileBytes + kDoStages * kTileBytes + kDsBytes +
                                    kDqStages * kDqChunkBytes + kQStages * kVecBytes + 8 * kNumBars + 16;
  static constexpr int kThreads = 512;
  static constexpr bool kAliasDq = (D == 128);
  static constexpr uint32_t kColS = 0, kColDP = 128, kColDV = 256, kColDK = 256 + D;
  static constexpr uint32_t kColDQ = kAliasDq ? 128 : 256 + 2 * D;
  // Exponentials all on the special-function unit: the polynomial on the FMA
  // pipe costs more issue slots than it frees here (measured at D = 64 and 128).
  static constexpr bool kPolyExp = false;
};
static_assert(BwdCfg<128>::kSmemBytes <= 232448 && BwdCfg<64>::kSmemBytes <= 232448,
              "backward shared memory over the per-CTA limit");
// Per-thread register budgets after setmaxnreg (compute, compute, drain, MMA +
// producers): an increase waits until decreases have freed the registers, so
// the four must add up to the 4 x 128 the 512-thread launch provides.
// The strided instantiations give the drain more: its epilogue also addresses
// rows itself (packed sequences that end inside a key tile).
template <bool kStrided>
struct BwdRegs {
  static constexpr int kCompute = kStrided ? 128 : 136, kDrain = kStrided ? 160 : 144, kOther = 96;
  static_assert(2 * kCompute + kDrain + kOther == 4 * 128, "register split must sum to the launch");
};

// ---------------------------------------------------------------- preprocess
// Half a warp per row (16 lanes x 16 bytes of O and of dO for D = 128, two rows
// per warp instruction), four rows per warp, eight warps per block: wide
// enough loads to keep HBM busy on this memory-bound pass.
constexpr int kPreRowsPerWarp = 4;

template <int D, bool kStrided = false>
__global__ void __launch_bounds__(256) bwd_pre_kernel(const BwdArgs<kStrided> p) {
  constexpr int kLanesPerRow = D / 8;             // 8 bf16 (16 bytes) per lane
  constexpr int kRowsPerPass = 32 / kLanesPerRow;  // 2 (D = 128) or 4 (D = 64)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sub = lane / kLanesPerRow, part = lane % kLanesPerRow;
  bool packed = false;
  if constexpr (kStrided) packed = p.rowoff != nullptr;
  // workspace rows: B*H*Np, or (packed) H*tp
  size_t rows = static_cast<size_t>(p.B) * p.H * p.Np;
  if constexpr (kStrided)
    if (packed) rows = static_cast<size_t>(p.H) * p.tp;
  const size_t row0 = (static_cast<size_t>(blockIdx.x) * 8 + warp) * kPreRowsPerWarp;
  // packed: the block's 32 rows lie in one 128-row tile, so in one sequence
  // (found once, by every warp as a whole)
  int pb = 0;
  if constexpr (kStrided)
    if (packed) pb = packed_seq_of_ws_row(p, static_cast<int>((static_cast<size_t>(blockIdx.x) * 32) % p.tp));
#pragma unroll
  for (int pass = 0; pass < kPreRowsPerWarp / kRowsPerPass; ++pass) {
    const size_t row = row0 + pass * kRowsPerPass + sub;  // over the workspace rows
    const bool in = row < rows;
    size_t bh = in ? row / p.Np : 0;
    int n = in ? static_cast<int>(row % p.Np) : 0;
    int len = 0, rb = 0;  // packed: the sequence's length and first row
    if constexpr (kStrided) {
      if (packed && in) {
        const int h = static_cast<int>(row / p.tp), R = static_cast<int>(row % p.tp);
        const int b = pb;
        packed_range(p, b, rb, len);
        n = R - packed_ws_row(rb, b);
        bh = static_cast<size_t>(b) * p.H + h;
      }
    }
    // Zero D floats of the dQ accumulator: linear rows 128t .. 128t + 127 cover
    // exactly the floats of its 128-row tile t, whatever the order inside the
    // tile.  Packed: tiles of a sequence's gap rows are never touched again.
    bool zero = in;
    if constexpr (kStrided)
      if (packed) zero = in && !p.dq_first_store && n >= 0 && n / 128 * 128 < len;
    if (zero) {
      float4* acc = reinterpret_cast<float4*>(p.dqacc + row * D);
      acc[2 * part] = make_float4(0.f, 0.f, 0.f, 0.f);
      acc[2 * part + 1] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    const bool valid = in && n >= 0 && n < (packed ? len : valid_rows(p, static_cast<int>(bh / p.H)));
    float s = 0.f;
    if (valid) {
      const __nv_bfloat16* orow;
      const __nv_bfloat16* drow;
      if constexpr (kStrided) {
        const int b = static_cast<int>(bh / p.H), h = static_cast<int>(bh % p.H);
        const int bi = packed ? 0 : b, ni = packed ? rb + n : n;  // packed: one batch entry of T rows
        orow = static_cast<const __nv_bfloat16*>(p.o) + p.so.row(bi, h, ni);
        drow = static_cast<const __nv_bfloat16*>(p.dout) + p.sdo.row(bi, h, ni);
      } else {
        orow = static_cast<const __nv_bfloat16*>(p.o) + (bh * p.N + n) * D;
        drow = static_cast<const __nv_bfloat16*>(p.dout) + (bh * p.N + n) * D;
      }
      const uint4 a = reinterpret_cast<const uint4*>(orow)[part];
      const uint4 c = reinterpret_cast<const uint4*>(drow)[part];
      const uint32_t av[4] = {a.x, a.y, a.z, a.w}, cv[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        s = fmaf(__uint_as_float(av[e] << 16), __uint_as_float(cv[e] << 16), s);
        s = fmaf(__uint_as_float(av[e] & 0xffff0000u), __uint_as_float(cv[e] & 0xffff0000u), s);
      }
    }
#pragma unroll
    for (int off = kLanesPerRow / 2; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    if (in && part == 0) {
      // tile padding or a padded token: D = 0 and LSE = +inf, so its P is exactly 0
      float lse = 0.f;
      if (valid) {
        const size_t h = bh % p.H;
        lse = packed ? p.lse[static_cast<size_t>(rb) * p.H + h * len + n] : p.lse[bh * p.N + n];
      }
      p.nD[row] = valid ? -s : 0.f;
      p.nlse2[row] = valid ? -lse * 1.4426950408889634f : -INFINITY;
    }
  }
}

// ---------------------------------------------------------------- dQ accumulator layout
// The partial dQ tile of one (query tile, key tile) pair is reduced as D / 32
// chunks of 128 rows x 32 columns (16 KB, contiguous in the accumulator so that
// one bulk reduce-add covers it).  Inside a chunk, row r holds its 32 floats in
// eight 16-byte units, unit u stored at position u ^ (r % 8): the drain's
// shared-memory writes (one row per thread) then spread over all banks.
// Tiles are numbered by workspace row / 128 (head bh's rows start at row
// bh * Np, or for packed sequences at h * tp + the sequence's start).  Element
// (row n, column c) sits at float index
//   dqacc_chunk<D>(n / 128, c / 32) + (n % 128) * 32
//     + (((c % 32) / 4) ^ (n % 8)) * 4 + c % 4.
template <int D>
__device__ __forceinline__ size_t dqacc_chunk(size_t tile, int chunk) {
  return (tile * (D / 32) + chunk) * 4096;
}

// ---------------------------------------------------------------- dQ convert
// One block per 32-row group: coalesced reads of the chunked accumulator, a
// transpose through shared memory, coalesced bf16 row writes of scale * acc.
template <int D, bool kStrided = false>
__global__ void __launch_bounds__(256) bwd_dq_kernel(const BwdArgs<kStrided> p) {
  __shared__ float tile[32][D + 4];
  // One block per 32 workspace rows: of head bh's Np rows, or (packed) of head
  // h's tp rows, where they belong to sequence b (rows past its end are skipped).
  int groups = p.Np / 32;
  bool packed = false;
  if constexpr (kStrided) {
    packed = p.rowoff != nullptr;
    if (packed) groups = p.tp / 32;
  }
  size_t bh = blockIdx.x / groups;
  const int g = static_cast<int>(blockIdx.x % groups);
  size_t tile0 = bh * p.ntiles;  // the accumulator's first 128-row tile of this head
  int nbase = 32 * g, nend = p.N, nvalid = 0, rb = 0;  // first row of the group, row limit, valid rows
  if constexpr (kStrided) {
    if (packed) {
      const int h = static_cast<int>(bh), b = packed_seq_of_ws_row(p, 32 * g);
      packed_range(p, b, rb, nvalid);
      nbase = 32 * g - packed_ws_row(rb, b);
      nend = nvalid;
      tile0 = static_cast<size_t>(h) * (p.tp / 128);
      bh = static_cast<size_t>(b) * p.H + h;
    }
  }
  if (!packed) nvalid = valid_rows(p, static_cast<int>(bh / p.H));
  if (packed && (nbase < 0 || nbase >= nend)) return;  // gap rows: nothing to convert
  const int t128 = g >> 2, r0 = (g & 3) * 32;  // 128-row tile and first row inside it
#pragma unroll
  for (int c = 0; c < D / 32; ++c) {  // 32 rows x 8 units of one chunk: 256 float4, one per thread
    const int rr = threadIdx.x >> 3, up = threadIdx.x & 7;
    const int u = up ^ (rr & 7);  // r0 is a multiple of 8, so (r0 + rr) % 8 = rr % 8
    const float4 a = reinterpret_cast<const float4*>(p.dqacc + dqacc_chunk<D>(tile0 + t128, c) +
                                                     static_cast<size_t>(r0) * 32)[threadIdx.x];
    *reinterpret_cast<float4*>(&tile[rr][c * 32 + 4 * u]) = a;
  }
  __syncthreads();
#pragma unroll
  for (int k = 0; k < D / 32; ++k) {
    const int f = threadIdx.x + 256 * k;
    const int rr = f / (D / 4), u = f % (D / 4);
    const int n = nbase + rr;
    if (n < 0 || n >= nend) continue;
    const float sc = n < nvalid ? p.scale : 0.f;
    uint2 out;
    out.x = pack_bf16x2(tile[rr][4 * u + 0] * sc, tile[rr][4 * u + 1] * sc);
    out.y = pack_bf16x2(tile[rr][4 * u + 2] * sc, tile[rr][4 * u + 3] * sc);
    long long at;
    if constexpr (kStrided)
      at = packed ? p.sdq.row(0, static_cast<int>(bh % p.H), rb + n) + 4 * u
                  : p.sdq.row(static_cast<int>(bh / p.H), static_cast<int>(bh % p.H), n) + 4 * u;
    else
      at = static_cast<long long>((bh * p.N + n) * D + 4 * u);
    *reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(p.dq) + at) = out;
  }
}

// Writes 32 fp32 values of row r (columns c..c+31 of a D-wide row), converted to
// bf16, into a 128-row tile staged in the TMA 128-byte-swizzled layout.
__device__ __forceinline__ void stage_row32_bf16(uint8_t* tile, int r, int c, const uint32_t (&v)[32], float mul) {
  const int chunk = c >> 6, u0 = (c & 63) >> 3;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    uint4 val;
    val.x = pack_bf16x2(__uint_as_float(v[8 * u + 0]) * mul, __uint_as_float(v[8 * u + 1]) * mul);
    val.y = pack_bf16x2(__uint_as_float(v[8 * u + 2]) * mul, __uint_as_float(v[8 * u + 3]) * mul);
    val.z = pack_bf16x2(__uint_as_float(v[8 * u + 4]) * mul, __uint_as_float(v[8 * u + 5]) * mul);
    val.w = pack_bf16x2(__uint_as_float(v[8 * u + 6]) * mul, __uint_as_float(v[8 * u + 7]) * mul);
    *reinterpret_cast<uint4*>(tile + chunk * 16384 + r * 128 + (((u0 + u) ^ (r & 7)) << 4)) = val;
  }
}

// P^T = 2^(S^T * scale_log2 - LSE_q * log2 e) for one key row and 64 query
// columns, in place (x holds the raw scores on entry, the weights on exit).
// The negated LSE values are broadcast from shared memory, 16 bytes per load.
// kPoly: one pair in four on the FMA pipe (exp2_poly2), unmasked tiles only.
template <bool kPoly>
__device__ __forceinline__ void exp_cols64(float (&x)[64], const float* nLv, float sl2) {
  const uint64_t sl2x2 = f2(sl2, sl2);
#pragma unroll
  for (int c4 = 0; c4 < 16; ++c4) {
    const float4 l4 = reinterpret_cast<const float4*>(nLv)[c4];
    float a0, a1, a2, a3;
    f2_split(ffma2(f2(x[4 * c4 + 0], x[4 * c4 + 1]), sl2x2, f2(l4.x, l4.y)), a0, a1);
    f2_split(ffma2(f2(x[4 * c4 + 2], x[4 * c4 + 3]), sl2x2, f2(l4.z, l4.w)), a2, a3);
    x[4 * c4 + 0] = fast_exp2(a0);
    x[4 * c4 + 1] = fast_exp2(a1);
    if (kPoly && (c4 & 1)) {
      exp2_poly2(a2, a3, x[4 * c4 + 2], x[4 * c4 + 3]);
    } else {
      x[4 * c4 + 2] = fast_exp2(a2);
      x[4 * c4 + 3] = fast_exp2(a3);
    }
  }
}

// ---------------------------------------------------------------- main kernel
// Work: slots numbered over (rasterisation group, slot, kv head), each holding
// one 128-key tile of one kv head, or under a causal mask two, key tiles j and
// ntiles - 1 - j, whose query-tile counts add up to the same total for every
// slot.  CTA c runs slots c, c + gridDim.x, c + 2 gridDim.x, ... (the grid is
// at most one CTA per SM), one job (key tile) after another, with every
// pipeline running on from one job into the next: the next job's Q and dO
// tiles load while the current one finishes, and its first products start
// while the drain warpgroup writes the current job's dK and dV.

template <int D, bool kMask, bool kStrided = false>
__global__ void __launch_bounds__(512, 1)
    bwd_sm100_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                     const __grid_constant__ CUtensorMap tmdK, const __grid_constant__ CUtensorMap tmdV,
                     const BwdArgs<kStrided> p) {
  using C = BwdCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (smem_u32(smem_raw) & 1023u) {  // layout below assumes a 1024-aligned window
    if (threadIdx.x == 0) atomicOr(&g_status, kStatusMisaligned);
    return;
  }
  uint8_t* sKV = smem_raw;                                 // K/V buffer kb: K at 2 kb kTileBytes, V after it
  uint8_t* sQ = smem_raw + 2 * C::kKvBufs * C::kTileBytes;  // Q stage s at s * kTileBytes
  uint8_t* sDO = sQ + C::kQStages * C::kTileBytes;        // dO stage s at s * kTileBytes
  uint8_t* sDS = sDO + C::kDoStages * C::kTileBytes;
  uint8_t* sDQ = sDS + C::kDsBytes;  // dQ staging buffers, kDqChunkBytes each; dK/dV epilogue staging
  uint8_t* sVec = sDQ + C::kDqStages * C::kDqChunkBytes;  // Q stage s: -LSE*log2(e) [128] then -D [128]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sVec + C::kQStages * C::kVecBytes);
  uint64_t* kv_full = bars;                 // per K/V buffer
  uint64_t* kv_empty = bars + C::kKvBufs;   // per K/V buffer: a job's products no longer read it
  uint64_t* q_full = bars + 2 * C::kKvBufs;
  uint64_t* q_empty = q_full + C::kQStages;
  uint64_t* do_full = q_empty + C::kQStages;
  uint64_t* do_empty = do_full + C::kDoStages;
  uint64_t* s_full = do_empty + C::kDoStages;
  uint64_t* dp_full = s_full + 1;
  uint64_t* p_full = s_full + 2;
  uint64_t* ds_full = s_full + 3;
  uint64_t* dq_full = s_full + 4;
  uint64_t* dq_empty = s_full + 5;
  uint64_t* kv_done = s_full + 6;    // a job's dV and dK are complete in TMEM
  uint64_t* acc_empty = s_full + 7;  // a job's dV and dK have been read out of TMEM
  uint64_t* mma_idle = s_full + 8;   // every product the MMA thread issued has completed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- this CTA's jobs.  Slots are numbered group-major: groups of p.group
  // kv heads run together (their Q, dO, K, V and dQ accumulator stay in L2).
  const int BHkv = p.B * p.Hkv;
  const int nslots = p.slots * BHkv;
  struct Job {
    int gs, sub;  // global slot, key tile within the slot
  };
  auto slot_of = [&](int gs, int& slot, int& bkv) {
    const int per_group = p.group * p.slots;
    const int grp = gs / per_group;
    const int g0 = grp * p.group;
    const int gsz = min(p.group, BHkv - g0);
    const int rem = gs - grp * per_group;
    slot = rem / gsz;
    bkv = g0 + rem % gsz;
  };
  bool packed = false;
  if constexpr (kStrided) packed = p.rowoff != nullptr;
  // Packed (one slot per sequence and kv head): the slot's key tiles one after
  // another, j = sub, so the sequence's Q, dO and dQ accumulator tiles stay in
  // L2 between its jobs.
  auto tile_of = [&](Job J, int slot) {
    return packed ? J.sub : (p.pairs ? (J.sub == 0 ? slot : p.ntiles - 1 - slot) : slot);
  };
  auto job_step = [&](Job J) {
    int slot, bkv;
    slot_of(J.gs, slot, bkv);
    if (packed ? J.sub + 1 < p.ntiles : (J.sub == 0 && p.pairs && p.ntiles - 1 - slot != slot))
      return Job{J.gs, J.sub + 1};
    return Job{J.gs + static_cast<int>(gridDim.x), 0};
  };
  // Packed: a key tile past its sequence's end is no job at all (its rows
  // belong to the next sequence, so nothing is stored for it).
  auto job_skip = [&](Job J) {
    if constexpr (kStrided) {
      if (packed) {
        int slot, bkv, rb, len;
        slot_of(J.gs, slot, bkv);
        const int j = tile_of(J, slot);
        packed_range(p, bkv / p.Hkv, rb, len);
        return j * 128 >= len;
      }
    }
    return false;
  };
  auto job_next = [&](Job J) {
    do {
      J = job_step(J);
    } while (J.gs < nslots && job_skip(J));
    return J;
  };
  Job job0{static_cast<int>(blockIdx.x), 0};
  if (job0.gs < nslots && job_skip(job0)) job0 = job_next(job0);
  // One job: key tile j of kv head bkv, its query-tile range [ilo, ihi] and the
  // number of (query head, query tile) work items.  Work items are walked in
  // increasing order, skipping blocks a block-sparse mask switches off; every
  // role walks the same jobs and items with its own cursors, so all roles see
  // the same sequence.  (kMask: the block-sparse variant; the dense kernels
  // compile no mask test.)
  struct Unit {
    int j, k0, ilo, ihi, total;
    int bkv, b, kh, bh0, Lb;  // kv head, batch entry, kv head in it, first query head, valid rows
    int rb, cb, ckv, cq0;     // tensor-map coordinates: first row, batch entry, kv head, first query head
    size_t w0;                // workspace row of (first query head, row 0); query head hq adds hq * wstride
  };
  size_t wstride = p.Np;  // workspace rows per query head
  if constexpr (kStrided)
    if (packed) wstride = p.tp;
  struct QCursor {
    int hq, i;
  };
  auto active = [&](const Unit& U, int hq, int i) {
    return !kMask || p.bmask[(U.bh0 + hq) * p.bmask_hs + static_cast<long long>(i) * p.ntiles + U.j] != 0;
  };
  auto advance = [&](const Unit& U, QCursor c) {  // next active item strictly after c
    do {
      if (++c.i > U.ihi) {
        c.i = U.ilo;
        ++c.hq;
      }
    } while (kMask && c.hq < p.g && !active(U, c.hq, c.i));
    return c;
  };
  auto first = [&](const Unit& U) {
    QCursor c{0, U.ilo};
    if (kMask && !active(U, 0, U.ilo)) c = advance(U, c);
    return c;
  };
  auto unit = [&](Job J) {
    Unit U;
    int slot;
    slot_of(J.gs, slot, U.bkv);
    U.b = U.bkv / p.Hkv;
    U.kh = U.bkv % p.Hkv;
    U.Lb = valid_rows(p, U.b);
    U.bh0 = U.b * p.H + U.kh * p.g;
    U.rb = 0;
    U.cb = U.b;
    U.ckv = U.bkv;
    U.cq0 = U.bh0;
    U.w0 = static_cast<size_t>(U.bh0) * p.Np;
    if constexpr (kStrided) {
      if (packed) {  // one batch entry of T rows in the maps; the sequence starts at row rb
        packed_range(p, U.b, U.rb, U.Lb);
        U.cb = 0;
        U.ckv = U.kh;
        U.cq0 = U.kh * p.g;
        U.w0 = static_cast<size_t>(U.kh * p.g) * p.tp + packed_ws_row(U.rb, U.b);
      }
    }
    U.j = tile_of(J, slot);
    U.k0 = U.j * 128;
    U.ilo = 0;
    U.ihi = (max(U.Lb, 1) - 1) / 128;  // query tiles holding valid rows
    if (p.causal) U.ilo = U.j;
    if (p.window >= 0) {
      U.ilo = max(U.ilo, max(0, U.k0 - p.window) / 128);
      U.ihi = min(U.ihi, (U.k0 + 127 + p.window) / 128);
    }
    const bool no_work = U.ilo > U.ihi || U.k0 >= U.Lb;  // nothing reaches this key tile
    U.total = no_work ? 0 : (U.ihi - U.ilo + 1) * p.g;
    if (kMask && !no_work) {
      U.total = 0;
      for (QCursor c = first(U); c.hq < p.g; c = advance(U, c)) ++U.total;
    }
    return U;
  };

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kKvBufs; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    for (int i = 0; i < C::kQStages; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
    }
    for (int i = 0; i < C::kDoStages; ++i) {
      mbar_init(&do_full[i], 1);
      mbar_init(&do_empty[i], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(dp_full, 1);
    mbar_init(p_full, 256);
    mbar_init(ds_full, 256);
    mbar_init(dq_full, 1);
    mbar_init(dq_empty, 128);
    mbar_init(kv_done, 1);
    mbar_init(acc_empty, 128);
    mbar_init(mma_idle, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 12) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
#ifdef FA_TRACE
  if (threadIdx.x == 0) {
    FA_TRACE_AT(6, 0, 0);
    uint32_t smid;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
    int items = 0;
    for (Job J = job0; J.gs < nslots; J = job_next(J)) items += unit(J).total;
    FA_TRACE_CTA(0, smid);
    FA_TRACE_CTA(1, items);
    FA_TRACE_CTA(2, globaltimer_ns());
  }
#endif

  if (warp >= 12) {
    regs_dec<BwdRegs<kStrided>::kOther>();
    if (warp == 13 && lane == 0) {
      // ---------------------------------------------------------- producer: K, V, Q + LSE + D
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      const bool stall = g_debug_stall != 0;  // test hook: the first K/V never arrive
      int issued[C::kQStages], kv_issued[C::kKvBufs];
#pragma unroll
      for (int i = 0; i < C::kQStages; ++i) issued[i] = 0;
#pragma unroll
      for (int i = 0; i < C::kKvBufs; ++i) kv_issued[i] = 0;
      int git = 0, u = 0;
      bool ok = true;
      for (Job J = job0; ok && J.gs < nslots; J = job_next(J), ++u) {
        const Unit U = unit(J);
        const int kb = u % C::kKvBufs;
        // K and V of this job replace those of job u - kKvBufs once its products are done with them
        if (u >= C::kKvBufs && !(ok = mbar_wait(&kv_empty[kb], (u / C::kKvBufs - 1) & 1, abort_flag))) break;
        if (!(stall && u == 0)) {
          uint8_t* sK = sKV + kb * 2 * C::kTileBytes;
          uint8_t* sV = sK + C::kTileBytes;
          mbar_arrive_expect_tx(&kv_full[kb], 2 * C::kTileBytes);
          for (int c = 0; c < C::kChunks; ++c) {
            if constexpr (kStrided) {
              tma_load_tile(&tmK, p.map4 & kBMapK, &kv_full[kb], sK + c * 16384, c * 64, U.rb + U.k0, U.ckv, U.kh,
                            U.cb);
              tma_load_tile(&tmV, p.map4 & kBMapV, &kv_full[kb], sV + c * 16384, c * 64, U.rb + U.k0, U.ckv, U.kh,
                            U.cb);
            } else {
              tma_load_3d(&tmK, &kv_full[kb], sK + c * 16384, c * 64, U.k0, U.bkv);
              tma_load_3d(&tmV, &kv_full[kb], sV + c * 16384, c * 64, U.k0, U.bkv);
            }
          }
          ++kv_issued[kb];
        }
        QCursor cur = first(U);
        for (int it = 0; it < U.total; ++it, ++git, cur = advance(U, cur)) {
          const int s = git % C::kQStages;
          if (!(ok = mbar_wait(&q_empty[s], ((git / C::kQStages) & 1) ^ 1, abort_flag))) break;
          FA_TRACE_AT(5, git, 0);
          mbar_arrive_expect_tx(&q_full[s], C::kTileBytes + C::kVecBytes);
          const int row0 = cur.i * 128, bh = U.bh0 + cur.hq;
          uint8_t* st = sQ + s * C::kTileBytes;
          for (int c = 0; c < C::kChunks; ++c) {
            if constexpr (kStrided)
              tma_load_tile(&tmQ, p.map4 & kBMapQ, &q_full[s], st + c * 16384, c * 64, U.rb + row0, U.cq0 + cur.hq,
                            U.kh * p.g + cur.hq, U.cb);
            else
              tma_load_3d(&tmQ, &q_full[s], st + c * 16384, c * 64, row0, bh);
          }
          const size_t vrow = U.w0 + cur.hq * wstride + row0;
          bulk_load(sVec + s * C::kVecBytes, p.nlse2 + vrow, 512, &q_full[s]);
          bulk_load(sVec + s * C::kVecBytes + 512, p.nD + vrow, 512, &q_full[s]);
          ++issued[s];
        }
      }
      // Never leave the CTA with copies still landing in shared memory.
      for (int kb = 0; kb < C::kKvBufs; ++kb)
        if (kv_issued[kb] > 0) mbar_wait_drain(&kv_full[kb], (kv_issued[kb] - 1) & 1);
      for (int s = 0; s < C::kQStages; ++s)
        if (issued[s] > 0) mbar_wait_drain(&q_full[s], (issued[s] - 1) & 1);
    } else if (warp == 15 && lane == 0) {
      // ---------------------------------------------------------- producer: dO
      prefetch_tmap(&tmdO);
      int issued[C::kDoStages];
#pragma unroll
      for (int i = 0; i < C::kDoStages; ++i) issued[i] = 0;
      int git = 0;
      bool ok = true;
      for (Job J = job0; ok && J.gs < nslots; J = job_next(J)) {
        const Unit U = unit(J);
        QCursor cur = first(U);
        for (int it = 0; it < U.total; ++it, ++git, cur = advance(U, cur)) {
          const int s = git % C::kDoStages;
          if (!(ok = mbar_wait(&do_empty[s], ((git / C::kDoStages) & 1) ^ 1, abort_flag))) break;
          FA_TRACE_AT(5, git, 1);
          mbar_arrive_expect_tx(&do_full[s], C::kTileBytes);
          const int row0 = cur.i * 128, bh = U.bh0 + cur.hq;
          uint8_t* st = sDO + s * C::kTileBytes;
          for (int c = 0; c < C::kChunks; ++c) {
            if constexpr (kStrided)
              tma_load_tile(&tmdO, p.map4 & kBMapDO, &do_full[s], st + c * 16384, c * 64, U.rb + row0,
                            U.cq0 + cur.hq, U.kh * p.g + cur.hq, U.cb);
            else
              tma_load_3d(&tmdO, &do_full[s], st + c * 16384, c * 64, row0, bh);
          }
          ++issued[s];
        }
      }
      for (int s = 0; s < C::kDoStages; ++s)
        if (issued[s] > 0) mbar_wait_drain(&do_full[s], (issued[s] - 1) & 1);
    } else if (warp == 12 && lane == 0) {
      // ---------------------------------------------------------- MMA issuer
      // One thread issues every product in a fixed order, so that the tensor
      // pipe works on the critical chain first:
      //   ... dK_i, dQ_i, [dQ_i drained] dP^T_{i+1}, [P_{i+1} ready] dV_{i+1}, S^T_{i+2}, ...
      // dV and the next S^T then run while the compute warps form dS, and the
      // next dP^T is never queued behind them.  The chain runs on from one unit
      // into the next.
      const uint32_t aKV = smem_u32(sKV), aQ = smem_u32(sQ), aDO = smem_u32(sDO), aDS = smem_u32(sDS);
      constexpr uint32_t kIdS = idesc_bf16_f32(128, 128, false, false);  // S^T, dP^T
      constexpr uint32_t kIdG = idesc_bf16_f32(128, D, false, true);     // dV, dK (A from TMEM)
      constexpr uint32_t kIdQ = idesc_bf16_f32(128, D, true, true);      // dQ = dS K
      auto st_q = [&](int s) { return aQ + s * C::kTileBytes; };
      auto st_do = [&](int s) { return aDO + s * C::kTileBytes; };
      // X^T = A B^T with both operands K-major: A = K or V (rows = keys), B = Q or dO.
      auto kmajor_nt = [&](uint32_t dcol, uint32_t a, uint32_t bb) {
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t off = (k >> 2) * 16384 + (k & 3) * 32;
          umma_ss(tmem + dcol, sdesc_sw128(a + off, 16, 1024), sdesc_sw128(bb + off, 16, 1024), kIdS, k > 0);
        }
      };
      // acc += X^T(tmem, packed bf16, keys x queries) * B(smem, queries x D, MN-major)
      auto ts_acc = [&](uint32_t dcol, uint32_t acol, uint32_t bb, bool acc) {
#pragma unroll
        for (int k = 0; k < 8; ++k)
          umma_ts(tmem + dcol, tmem + acol + (k >> 2) * 64 + (k & 3) * 8,
                  sdesc_sw128(bb + k * 2048, 16384, 1024), kIdG, acc || k > 0);
      };
      bool ok = true;
      int git = 0;  // work items of the CTA before the current one (barrier phases run on across jobs)
      int u = 0;    // jobs of the CTA before the current one
      for (Job J = job0; ok && J.gs < nslots; J = job_next(J), ++u) {
        const Unit U = unit(J);
        const int kb = u % C::kKvBufs;
        const uint32_t aK = aKV + kb * 2 * C::kTileBytes, aV = aK + C::kTileBytes;
        if (!(ok = mbar_wait(&kv_full[kb], (u / C::kKvBufs) & 1, abort_flag))) break;
        if (U.total > 0) {
          if (!(ok = mbar_wait(&q_full[git % C::kQStages], (git / C::kQStages) & 1, abort_flag))) break;
          tc_fence_after();
          kmajor_nt(C::kColS, aK, st_q(git % C::kQStages));  // S^T of the first query tile
          umma_commit(s_full);
          if (C::kAliasDq && git > 0) {  // the previous unit's last dQ tile shares the dP^T columns
            if (!(ok = mbar_wait(dq_empty, (git - 1) & 1, abort_flag))) break;
          }
          if (!(ok = mbar_wait(&do_full[git % C::kDoStages], (git / C::kDoStages) & 1, abort_flag))) break;
          tc_fence_after();
          kmajor_nt(C::kColDP, aV, st_do(git % C::kDoStages));  // dP^T of the first query tile
          umma_commit(dp_full);
        }
        for (int it = 0; ok && it < U.total; ++it) {
          const int g = git + it;
          const int s = g % C::kQStages, s1 = (g + 1) % C::kQStages;
          const int so = g % C::kDoStages, so1 = (g + 1) % C::kDoStages;
          if (!(ok = mbar_wait(p_full, g & 1, abort_flag))) break;
          if (it == 0 && u > 0) {  // the accumulators start afresh: the previous unit's were read out
            if (!(ok = mbar_wait(acc_empty, (u - 1) & 1, abort_flag))) break;
          }
          FA_TRACE_AT(2, g, 0);
          tc_fence_after();
          ts_acc(C::kColDV, C::kColS, st_do(so), it > 0);  // dV += P^T dO (dO_i landed before dP^T_i)
          umma_commit(&do_empty[so]);                       // dP^T_i and dV_i have read dO_i
          FA_TRACE_AT(2, g, 1);
          if (it + 1 < U.total) {
            if (!(ok = mbar_wait(&q_full[s1], ((g + 1) / C::kQStages) & 1, abort_flag))) break;
            FA_TRACE_AT(2, g, 2);
            tc_fence_after();
            kmajor_nt(C::kColS, aK, st_q(s1));  // S^T of the next query tile
            umma_commit(s_full);
            FA_TRACE_AT(2, g, 3);
          }
          if (!(ok = mbar_wait(ds_full, g & 1, abort_flag))) break;
          FA_TRACE_AT(3, g, 0);
          tc_fence_after();
          ts_acc(C::kColDK, C::kColDP, st_q(s), it > 0);  // dK += dS^T Q
          if (!C::kAliasDq && g > 0) {
            if (!(ok = mbar_wait(dq_empty, (g - 1) & 1, abort_flag))) break;
            tc_fence_after();
          }
#pragma unroll
          for (int k = 0; k < 8; ++k)  // dQ_i = dS K (both operands MN-major in smem)
            umma_ss(tmem + C::kColDQ, sdesc_sw128(aDS + k * 2048, 16384, 1024),
                    sdesc_sw128(aK + k * 2048, 16384, 1024), kIdQ, k > 0);
          umma_commit(dq_full);
          umma_commit(&q_empty[s]);
          FA_TRACE_AT(3, g, 1);
          if (it + 1 < U.total) {
            if (C::kAliasDq) {  // the dQ tile shares the dP^T columns
              if (!(ok = mbar_wait(dq_empty, g & 1, abort_flag))) break;
            }
            if (!(ok = mbar_wait(&do_full[so1], ((g + 1) / C::kDoStages) & 1, abort_flag))) break;
            FA_TRACE_AT(3, g, 2);
            tc_fence_after();
            kmajor_nt(C::kColDP, aV, st_do(so1));  // dP^T of the next query tile
            umma_commit(dp_full);
            FA_TRACE_AT(3, g, 3);
          }
        }
        if (!ok) break;
        if (U.total == 0 && u > 0) {
          // A unit without products must still not complete its kv_done phase
          // before the drain has consumed the previous one (a waiter on a
          // phase parity must never be overtaken by two phases).
          if (!(ok = mbar_wait(acc_empty, (u - 1) & 1, abort_flag))) break;
        }
        git += U.total;
        umma_commit(&kv_empty[kb]);  // K and V may be replaced once these products complete
        umma_commit(kv_done);        // dV and dK of the job are complete
      }
      // Before the CTA frees TMEM: every product this thread issued has completed.
      umma_commit(mma_idle);
      mbar_wait_drain(mma_idle, 0);
    }
    __syncwarp();
  } else if (warp < 8) {
    // ------------------------------------------------------------ P and dS
    regs_inc<BwdRegs<kStrided>::kCompute>();
    // Warpgroup w handles query columns [64w, 64w + 64); one key row per thread.
    const int w = warp >> 2, wl = warp & 3;
    const int r = wl * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(wl * 32) << 16;
    const uint32_t tS = tmem + lane_off + C::kColS + 64 * w;
    const uint32_t tDP = tmem + lane_off + C::kColDP + 64 * w;
    const float sl2 = p.scale_log2;
    const int ds_chunk = w;  // 64-column (128-byte) block of the dS tile
    bool ok = true;
    int git = 0;
    for (Job J = job0; ok && J.gs < nslots; J = job_next(J)) {
      const Unit U = unit(J);
      const int key = U.k0 + r;
      const bool tile_valid = U.k0 + 127 < U.Lb;  // no padded key in this key tile
      const bool key_valid = key < U.Lb;
      QCursor cur = first(U);
      for (int it = 0; it < U.total; ++it, cur = advance(U, cur)) {
        const int g = git + it;
        const int s = g % C::kQStages;
        const int q0 = cur.i * 128 + 64 * w;  // first query of my columns
        const float* nLv = reinterpret_cast<const float*>(sVec + s * C::kVecBytes) + 64 * w;
        const float* nDv = reinterpret_cast<const float*>(sVec + s * C::kVecBytes + 512) + 64 * w;
        bool full = tile_valid;  // every (query, key) pair of my 64 columns allowed?
        if (p.causal) full = full && (U.k0 + 127 <= q0);
        if (p.window >= 0) full = full && (q0 + 63 - U.k0 <= p.window) && (U.k0 + 127 - q0 <= p.window);
        // (warp-uniform outcomes: the TMEM loads and stores below are warp-collective)
        ok = mbar_wait(&q_full[s], (g / C::kQStages) & 1, abort_flag);  // LSE / D landed
        ok = ok && mbar_wait(s_full, g & 1, abort_flag);
        if (!(ok = __all_sync(0xffffffffu, ok))) break;
        if (lane == 0 && wl == 0) FA_TRACE_AT(w, g, 0);
        tc_fence_after();
        float pv[64];  // the fp32 weights P^T of my 64 columns
        {
          uint32_t sv[64];
          tmem_ld32(tS, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
          tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 64; ++c) pv[c] = __uint_as_float(sv[c]);
        }
        if (full && C::kPolyExp)
          exp_cols64<true>(pv, nLv, sl2);
        else
          exp_cols64<false>(pv, nLv, sl2);
        if (!full) {
          // Tiles on the diagonal / window edge only: my key row may see query
          // columns [c_lo, c_hi] of my 64; one unsigned compare per element.
          int c_lo = 0, c_hi = key_valid ? 63 : -1;
          if (p.causal) c_lo = max(c_lo, key - q0);
          if (p.window >= 0) {
            c_lo = max(c_lo, key - p.window - q0);
            c_hi = min(c_hi, key + p.window - q0);
          }
          if (c_hi < c_lo) c_lo = 64, c_hi = 64;  // nothing allowed: (c - 64) wraps above the span
          const uint32_t span = static_cast<uint32_t>(c_hi - c_lo);
#pragma unroll
          for (int c = 0; c < 64; ++c) pv[c] = static_cast<uint32_t>(c - c_lo) <= span ? pv[c] : 0.f;
        }
        {
          uint32_t pk[32];  // my 64 P^T values, packed bf16: the A operand of dV += P^T dO
#pragma unroll
          for (int c2 = 0; c2 < 32; ++c2) pk[c2] = pack_bf16x2(pv[2 * c2], pv[2 * c2 + 1]);
          tmem_st32(tS, pk);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(p_full);
        if (lane == 0 && wl == 0) FA_TRACE_AT(w, g, 1);

        ok = mbar_wait(dp_full, g & 1, abort_flag);
        if (!(ok = __all_sync(0xffffffffu, ok))) break;
        if (lane == 0 && wl == 0) FA_TRACE_AT(w, g, 2);
        tc_fence_after();
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t dv[32];
          tmem_ld32(tDP + 32 * h, dv);
          tmem_wait_ld();
          uint32_t ds[16];
#pragma unroll
          for (int u2 = 0; u2 < 8; ++u2) {
            const float4 d4 = reinterpret_cast<const float4*>(nDv)[8 * h + u2];
            // dS = P (dP - D) on packed pairs, P kept in fp32 since the exponent phase
            const int c = 32 * h + 4 * u2;
            float a0, a1, a2, a3;
            f2_split(fmul2(f2(pv[c], pv[c + 1]),
                           fadd2(f2(__uint_as_float(dv[4 * u2]), __uint_as_float(dv[4 * u2 + 1])), f2(d4.x, d4.y))),
                     a0, a1);
            f2_split(fmul2(f2(pv[c + 2], pv[c + 3]), fadd2(f2(__uint_as_float(dv[4 * u2 + 2]),
                                                              __uint_as_float(dv[4 * u2 + 3])),
                                                           f2(d4.z, d4.w))),
                     a2, a3);
            ds[2 * u2] = pack_bf16x2(a0, a1);
            ds[2 * u2 + 1] = pack_bf16x2(a2, a3);
          }
          // dS^T (packed) over dP^T columns this thread has already read; dS into
          // shared memory as rows = keys, columns = queries (MN-major A of dQ).
          tmem_st16(tDP + 16 * h, ds);
#pragma unroll
          for (int u4 = 0; u4 < 4; ++u4) {
            const int unit16 = h * 4 + u4;  // 16-byte unit within my 128-byte row chunk
            *reinterpret_cast<uint4*>(sDS + ds_chunk * 16384 + r * 128 + ((unit16 ^ (r & 7)) << 4)) =
                make_uint4(ds[4 * u4], ds[4 * u4 + 1], ds[4 * u4 + 2], ds[4 * u4 + 3]);
          }
        }
        tmem_wait_st();
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(ds_full);
        if (lane == 0 && wl == 0) FA_TRACE_AT(w, g, 3);
      }
      git += U.total;
    }
  } else {
    // ------------------------------------------------------------ dQ drain and the dK/dV epilogue
    regs_inc<BwdRegs<kStrided>::kDrain>();
    const int wl = warp & 3;
    const int r = wl * 32 + lane;  // query row of the dQ tile (drain), key row (epilogue)
    const uint32_t lane_off = static_cast<uint32_t>(wl * 32) << 16;
    constexpr int kBarDrain = 1, kBarDrainAnd = 2;  // named barriers of the 128 drain threads
    bool ok = true;
    int nchunk = 0;  // chunks handed to the TMA unit so far
    int git = 0, u = 0;
    for (Job J = job0; ok && J.gs < nslots; J = job_next(J), ++u) {
      const Unit U = unit(J);
      bool first_store = false;  // this job writes the first dQ partial of each of its tiles
      if constexpr (kStrided) first_store = packed && p.dq_first_store && U.j == 0;
      QCursor cur = first(U);
      for (int it = 0; it < U.total; ++it, cur = advance(U, cur)) {
        const int g = git + it;
        ok = mbar_wait(dq_full, g & 1, abort_flag);
        // all 128 threads take the same branch: the named barriers below need every one of them
        if (!(ok = named_bar_and(kBarDrainAnd, 128, ok))) break;
        if (r == 0) FA_TRACE_AT(4, g, 0);
        tc_fence_after();
        uint32_t v[D];
#pragma unroll
        for (int c = 0; c < D / 32; ++c)
          tmem_ld32(tmem + lane_off + C::kColDQ + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&v[c * 32]));
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(dq_empty);  // TMEM tile free before the reductions are staged
        if (r == 0) FA_TRACE_AT(4, g, 1);
        // the accumulator's first 128-row tile of this query head
        const size_t tile0 = (U.w0 + cur.hq * wstride) / 128;
#pragma unroll
        for (int c = 0; c < C::kDqChunks; ++c, ++nchunk) {
          uint8_t* buf = sDQ + (nchunk % C::kDqStages) * C::kDqChunkBytes;
          // the buffer's previous chunk has been read by the TMA unit
          if (r == 0 && nchunk >= C::kDqStages) bulk_wait_read<C::kDqStages - 1>();
          named_bar_sync(kBarDrain, 128);
#pragma unroll
          for (int u8 = 0; u8 < 8; ++u8)
            *reinterpret_cast<uint4*>(buf + r * 128 + ((u8 ^ (r & 7)) << 4)) =
                make_uint4(v[c * 32 + 4 * u8], v[c * 32 + 4 * u8 + 1], v[c * 32 + 4 * u8 + 2],
                           v[c * 32 + 4 * u8 + 3]);
          fence_proxy_async_smem();
          named_bar_sync(kBarDrain, 128);
          if (r == 0) {
            float* dst = p.dqacc + dqacc_chunk<D>(tile0 + cur.i, c);
            if (first_store)
              bulk_store(dst, buf, C::kDqChunkBytes);
            else
              bulk_reduce_add_f32(dst, buf, C::kDqChunkBytes);
            bulk_commit();
          }
        }
        if (r == 0) FA_TRACE_AT(4, g, 2);
      }
      if (!ok) break;
      git += U.total;
      // ---- epilogue of the unit: dV and dK (x scale) to bf16, through the staging buffers
      ok = named_bar_and(kBarDrainAnd, 128, mbar_wait(kv_done, u & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      // staging buffers no longer read by earlier reductions (first-store job:
      // its stores complete, before the next jobs add into the same tiles)
      if (r == 0) {
        if (first_store)
          bulk_wait0();
        else
          bulk_wait_read0();
      }
      named_bar_sync(kBarDrain, 128);
      uint8_t* sDV = sDQ;                                  // bf16 128 x D tile in the TMA layout
      uint8_t* sDK = sDQ + (D == 128 ? 0 : C::kTileBytes);  // after dV's store has read it (D = 128)
      // Stores: the whole tile by the TMA unit, or (packed, the sequence ends
      // inside the key tile) each valid row by its own thread, or (packed, the
      // tile lies past the sequence end) nothing.
      const bool tma_out = !packed || U.k0 + 128 <= U.Lb;
      auto store_rows = [&](const uint8_t* sT, bool is_dk) {  // my row of a staged tile, if valid
        if constexpr (kStrided) {
          if (U.k0 + r < U.Lb) {
            __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(is_dk ? p.dk : p.dv) +
                                 static_cast<long long>(U.rb + U.k0 + r) * p.kv_rs +
                                 static_cast<long long>(U.kh) * p.kv_hs;
#pragma unroll
            for (int cc = 0; cc < D / 64; ++cc)
#pragma unroll
              for (int u8 = 0; u8 < 8; ++u8)
                *reinterpret_cast<uint4*>(dst + cc * 64 + u8 * 8) =
                    *reinterpret_cast<const uint4*>(sT + cc * 16384 + r * 128 + ((u8 ^ (r & 7)) << 4));
          }
        }
      };
#pragma unroll 1
      for (int c = 0; c < D; c += 32) {
        uint32_t t[32];
        if (U.total > 0) {
          tmem_ld32(tmem + lane_off + C::kColDV + c, t);
          tmem_wait_ld();
        } else {  // no query block reaches this key tile: dV = dK = 0
#pragma unroll
          for (int i = 0; i < 32; ++i) t[i] = 0u;
        }
        stage_row32_bf16(sDV, r, c, t, 1.f);
      }
      uint32_t v[D];  // dK row, held while dV's store reads the staging buffers
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        if (U.total > 0) {
          tmem_ld32(tmem + lane_off + C::kColDK + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&v[c * 32]));
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) v[c * 32 + i] = 0u;
        }
      }
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(acc_empty);  // the next unit's products may overwrite dV and dK
      fence_proxy_async_smem();
      named_bar_sync(kBarDrain, 128);
      if (r == 0 && tma_out) {
        for (int c = 0; c < C::kChunks; ++c) {
          if constexpr (kStrided)
            tma_store_tile(&tmdV, p.map4 & kBMapDV, sDV + c * 16384, c * 64, U.rb + U.k0, U.ckv, U.kh, U.cb);
          else
            tma_store_3d(&tmdV, sDV + c * 16384, c * 64, U.k0, U.bkv);
        }
        bulk_commit();
        if (D == 128) bulk_wait_read0();  // dK reuses the buffers dV's store reads
      }
      if (!tma_out) store_rows(sDV, false);
      named_bar_sync(kBarDrain, 128);
#pragma unroll
      for (int c = 0; c < D; c += 32)
        stage_row32_bf16(sDK, r, c, *reinterpret_cast<const uint32_t(*)[32]>(&v[c]), p.scale);
      fence_proxy_async_smem();
      named_bar_sync(kBarDrain, 128);
      if (r == 0 && tma_out) {
        for (int c = 0; c < C::kChunks; ++c) {
          if constexpr (kStrided)
            tma_store_tile(&tmdK, p.map4 & kBMapDK, sDK + c * 16384, c * 64, U.rb + U.k0, U.ckv, U.kh, U.cb);
          else
            tma_store_3d(&tmdK, sDK + c * 16384, c * 64, U.k0, U.bkv);
        }
        bulk_commit();
        bulk_wait_read0();  // the next unit's dQ chunks reuse the staging buffers
      }
      if (!tma_out) store_rows(sDK, true);
      named_bar_sync(kBarDrain, 128);
    }
    // Shared memory must outlive the copies that read it; the global side of the
    // reductions and stores completes with the grid.
    if (r == 0) bulk_wait_read0();
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) {
    FA_TRACE_AT(6, 0, 1);
    FA_TRACE_CTA(3, globaltimer_ns());
  }
  if (warp == 12) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace fa
