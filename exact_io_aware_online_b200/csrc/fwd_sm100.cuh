// fwd_sm100.cuh -- bf16 attention forward on sm_100a tensor cores.
//
// One CTA owns two 128-row query tiles of one (batch, head) and streams the
// head's K/V tiles (128 keys each) through a TMA ring in shared memory.  For
// every key tile it keeps, per query row, the online-softmax state of
// "Flash attention and efficient attention" (section "Derivation: Incremental
// Softmax"): the running maximum m, the running sum l and the unnormalised
// accumulator O~, rescaled when the maximum moves (Step 3's merge with one new
// block at a time).  Only O and the logsumexp reach global memory ("FlashAttention"
// guide page, "Tiling through SRAM").  Where units are short (a few key tiles
// each), fwd_persist_sm100.cuh runs the same tiles with CTAs that take unit
// after unit.
//
// Roles (384 threads, three warpgroups):
//   warps 0-3   softmax for query tile 0, one thread per row (TMEM lanes 0-127)
//   warps 4-7   softmax for query tile 1
//   warp 8      tcgen05.mma issuer (one thread) and TMEM owner
//   warp 9      TMA producer (one thread)
//   warps 10-11 idle (they complete the third warpgroup)
// Registers: 168 per thread at launch; the third warpgroup drops to 72 and the
// two softmax warpgroups rise to 216 (216 + 216 + 72 = 3 * 168), enough to hold
// a whole 128-key score row per thread without spilling.
// TMEM (512 columns): S0 [0,128) S1 [128,256) O0 [256,256+D) O1 [256+D,256+2D).
// P_t overwrites S_t as packed bf16 (64 columns) and is the A operand of the
// P V product straight from TMEM, so P never touches shared memory.
//
// Differences from the pages' own design (which is SRAM tiling for an older
// GPU): the scores live in TMEM, not registers or SRAM; exponentials are base 2
// with the scale folded in; and the rescale of O~ is lazy -- the reference
// maximum only moves when the new maximum exceeds it by more than kTau (log2
// units), which keeps every p <= 2^kTau and is exact after the final 1/l.
#pragma once

#include <type_traits>

#include "sm100_ptx.cuh"

namespace fa {

struct FwdParams {
  float* lse;
  int B, H, Hkv, N, g;
  float scale_log2;  // scale * log2(e)
  int causal, window;
  int npairs;     // ceil(N / 256): query-tile pairs per head
  int ntiles_kv;  // ceil(N / 128)
  int group;      // heads per rasterisation group (kept L2-resident together)
  // split-KV mode only: each CTA covers one of `splits` contiguous chunks of its
  // key-tile range and writes partial results instead of O and the logsumexp.
  int splits;
  int nq2;         // npairs * 256: rows per head in the partial buffers
  // block-sparse mode (non-null bmask): 0/1 per 128 x 128 block of the score
  // matrix, [query block][key block], nbt x nbt per query head at bmask_hs
  // elements apart (0: one mask for all heads).
  const uint8_t* bmask;
  long long bmask_hs;
  int nbt;
  float* part_o;   // [splits][B*H][nq2][D] fp32 unnormalised O~, lane-interleaved (fwd_part_index)
  float4* part_m;  // [splits][B*H][nq2] {m (log2 units), l, l_bf16, 0}
  // padded variable lengths (non-null): batch entry b has seqlens[b] valid rows;
  // later keys are masked and later query rows give O = 0, LSE = -inf.
  const int* seqlens;
};

// Arguments of the strided-layout instantiation: the same fields plus which
// tensor maps are 4-D (column, row, head, batch entry) rather than 3-D (column,
// row, batch entry * heads + head).  A separate type, so the contiguous
// instantiations keep the plain FwdParams.
struct FwdStridedParams : FwdParams {
  unsigned map4;
  // Packed variable lengths (non-null rowoff, device memory): batch entry b is
  // sequence b, rows rowoff[b] .. rowoff[b+1] - 1 of tensors that hold all T
  // rows back to back (one batch entry in the tensor maps); N is the longest
  // length.  Loads index from the sequence's first row; O rows are stored only
  // up to the sequence end (plain stores for a tile the end falls inside), and
  // the logsumexp of sequence b is [H, len_b] at lse + rowoff[b] * H.
  const int* rowoff;
  int T;
  void* o;
  long long o_rs, o_hs;  // element strides of O's rows and heads
};
constexpr unsigned kMapQ = 1, kMapK = 2, kMapV = 4, kMapO = 8;
// Arguments of the decode instantiation (split-KV only).  The g query heads
// that share a kv head are packed into one "virtual head" of g * nq rows (they
// are adjacent in memory), so H = Hkv and g = 1 in the base fields and a CTA
// reads each K/V tile once for the whole group.  Virtual row r is query
// r % nq of its head, at position qoff + r % nq with qoff = Nk - nq (the
// newest nq tokens of a length-Nk sequence).
struct FwdDecodeParams : FwdParams {
  int Nk, qoff, nq;
};

// Smallest and largest position of virtual rows r0..r1 (decode packing).
__device__ __forceinline__ void decode_positions(int r0, int r1, int nq, int qoff, int& pmin, int& pmax) {
  if (r1 - r0 + 1 >= nq || r0 % nq > r1 % nq) {  // every query position occurs
    pmin = qoff;
    pmax = qoff + nq - 1;
  } else {
    pmin = qoff + r0 % nq;
    pmax = qoff + r1 % nq;
  }
}
template <bool kStrided, bool kDecode = false>
using FwdArgs = std::conditional_t<kDecode, FwdDecodeParams, std::conditional_t<kStrided, FwdStridedParams, FwdParams>>;

// Partial-output layout: row n = 32 g + lane; the 16-byte unit u (columns
// 4u..4u+3) of 32 consecutive rows is contiguous, so a warp whose lane owns a
// row stores and loads 512 contiguous bytes per unit.
template <int D>
__device__ __forceinline__ size_t fwd_part_unit(size_t split_bh, int nq2, int g, int u) {
  return ((split_bh * static_cast<size_t>(nq2 / 32) + g) * (D / 4) + u) * 128;
}

template <int D>
struct FwdCfg {
  static constexpr int kTileBytes = 128 * D * 2;  // one 128-row bf16 tile
  static constexpr int kChunks = D / 64;          // 64-column (128-byte) chunks
  static constexpr int kStages = (D == 128) ? 4 : 8;
  static constexpr int kSmemQ = 2 * kTileBytes;
  static constexpr int kSmemKV = kStages * kTileBytes;
  static constexpr int kNumBars = 1 + 2 * kStages + 15;
  // P_t V is issued in kPvParts key ranges, each as soon as the softmax threads
  // have stored that range of P_t, so only the last range (and the next Q K^T)
  // sits between the end of the exponentials and the next score tile.  Two
  // halves pay at D = 64 (forward 5% faster at B=4 H=16 N=2048); at D = 128
  // the extra store wait in the exponent loop costs what the earlier half
  // saves (measured: equal or slower), so one range.
  static constexpr int kPvParts = (D == 64) ? 2 : 1;
  static constexpr int kSmemBytes = 1024 + kSmemQ + kSmemKV + 8 * kNumBars + 16;
  static constexpr int kThreads = 384;
  static constexpr uint32_t kTmemCols = 512;
  // A quarter of the exponentials on the FMA pipe (exp2_poly2) pays at D = 64,
  // where the special-function unit does twice the work per tensor-core cycle;
  // at D = 128 the extra instructions cost more than they save (measured).
  static constexpr bool kPolyExp = (D == 64);
};

constexpr float kTau = 8.0f;  // lazy-rescale threshold, log2 units (factor 256)
constexpr float kLn2 = 0.69314718055994530942f;

// p = 2^(s * scale_log2 - m) for one 128-key score row, written to TMEM as packed
// bf16 in four 32-key chunks; accumulates the fp32 row sum (l) and the sum of
// the bf16-rounded values (lb).  kPoly: one pair in four uses exp2_poly2 so
// the special-function unit is not the only source of exponentials.
template <bool kPoly, int kParts>
__device__ __forceinline__ void exp_row_to_tmem(const float (&s)[128], float sl2, float ms, uint32_t tS, float& l,
                                                float& lb, uint64_t* part_bar) {
  const uint64_t sl2x2 = f2(sl2, sl2), nmsx2 = f2(-ms, -ms);
  // Row sums on packed fp32 pairs, two independent accumulators each.  rs:
  // exact fp32 weights (gives the logsumexp); rsb: the bf16-rounded weights
  // the P V product actually uses, so O = sum(p v) / lb is a convex
  // combination of V rows even when one key dominates the row.
  uint64_t rs2[2] = {0ull, 0ull}, rsb2[2] = {0ull, 0ull};
#pragma unroll
  for (int ch = 0; ch < 4; ++ch) {  // 32 keys per chunk, stored as soon as packed
    uint32_t pk[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const int c = ch * 32 + 2 * u;
      float x0, x1, p0, p1;
      f2_split(ffma2(f2(s[c], s[c + 1]), sl2x2, nmsx2), x0, x1);
      if (kPoly && (u & 3) == 3) {
        exp2_poly2(x0, x1, p0, p1);
      } else {
        p0 = fast_exp2(x0);
        p1 = fast_exp2(x1);
      }
      pk[u] = pack_bf16x2(p0, p1);
      rs2[u & 1] = fadd2(rs2[u & 1], f2(p0, p1));
      rsb2[u & 1] = fadd2(rsb2[u & 1], f2(__uint_as_float(pk[u] << 16), __uint_as_float(pk[u] & 0xffff0000u)));
    }
    tmem_st16(tS + ch * 16, pk);
    if (kParts > 1 && ch < 3 && (ch + 1) % (4 / kParts) == 0) {  // this key range of P is in TMEM
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&part_bar[(ch + 1) / (4 / kParts) - 1]);
    }
  }
  float a0, a1, b0, b1;
  f2_split(fadd2(rs2[0], rs2[1]), a0, a1);
  f2_split(fadd2(rsb2[0], rsb2[1]), b0, b1);
  l += a0 + a1;
  lb += b0 + b1;
}

template <int D, bool kSplit, bool kMask, bool kStrided = false, bool kDecode = false>
__global__ void __launch_bounds__(384, 1)
    fwd_sm100_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                     const FwdArgs<kStrided, kDecode> p) {
  using C = FwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* base = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  uint8_t* sQ = base;
  uint8_t* sKV = base + C::kSmemQ;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sKV + C::kSmemKV);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;
  uint64_t* kv_empty = bars + 1 + C::kStages;
  uint64_t* s_full = bars + 1 + 2 * C::kStages;
  uint64_t* p_full = s_full + 2;
  uint64_t* o_full = s_full + 4;
  uint64_t* epi_bar = s_full + 6;  // softmax threads -> storing thread: O tile staged
  uint64_t* mma_idle = s_full + 8;  // every product the MMA thread issued has completed
  uint64_t* p_part = s_full + 9;    // [t * 3 + i]: softmax -> MMA, key range i of P_t stored (i < kPvParts - 1)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- work unit: query-tile pair `pair` of head bh.  Groups of p.group heads
  // run together (their K/V stay in L2); inside a group the heaviest (last)
  // pairs under a causal mask go first.
  const int BH = p.B * p.H;
  const int split = kSplit ? static_cast<int>(blockIdx.x) % p.splits : 0;
  const int unit = kSplit ? static_cast<int>(blockIdx.x) / p.splits : static_cast<int>(blockIdx.x);
  const int per_group = p.group * p.npairs;
  const int grp = unit / per_group;
  const int g0 = grp * p.group;
  const int gsz = min(p.group, BH - g0);
  const int rem = unit - grp * per_group;
  const int pair = p.npairs - 1 - rem / gsz;
  const int bh = g0 + rem % gsz;
  const int b = bh / p.H, h = bh % p.H;
  const int kvh = b * p.Hkv + h / p.g;
  const int q0 = pair * 256;
  int Lb = p.seqlens ? max(0, min(p.seqlens[b], p.N)) : p.N;  // valid rows of this batch entry
  // Tensor-map coordinates of this unit: first row, batch entry, head and kv head.
  int rb = 0, cb = b, cbh = bh, ckvh = kvh;
  bool packed = false;
  if constexpr (kStrided) {
    if (p.rowoff) {  // offsets clamped to the tensors' rows whatever they hold
      packed = true;
      rb = min(max(p.rowoff[b], 0), p.T);
      Lb = min(min(max(p.rowoff[b + 1], rb), p.T) - rb, p.N);
      cb = 0;
      cbh = h;
      ckvh = h / p.g;
    }
  }
  // Valid keys and the position of query row 0 (decode: Nk keys, queries are
  // the newest rows; otherwise the same rows as the queries, position 0).
  int Lk = Lb, qoff = 0;
  if constexpr (kDecode) {
    Lk = p.Nk;
    qoff = p.qoff;
  }
  const int qlast = min(q0 + 255, Lb - 1);
  int pmin = q0, pmax = qlast;  // positions of the pair's first and last valid rows
  if constexpr (kDecode) decode_positions(q0, qlast, p.nq, qoff, pmin, pmax);
  int jlo = 0, jhi = p.ntiles_kv - 1;
  jhi = min(jhi, (max(Lk, 1) - 1) / 128);  // key tiles holding valid rows
  if (p.causal) jhi = min(jhi, pmax / 128);
  if (p.window >= 0) {
    jlo = max(0, pmin - p.window) / 128;
    jhi = min(jhi, (pmax + p.window) / 128);
  }
  if (kSplit) {  // my contiguous chunk of the key-tile range (possibly empty)
    const int chunk = (jhi - jlo + p.splits) / p.splits;
    jlo += split * chunk;
    jhi = min(jhi, jlo + chunk - 1);
  }
  // Block-sparse: only key tiles whose block is on for either query tile are
  // visited (every role walks the same increasing sequence, see next_kv).
  // (kMask: the block-sparse variant; the dense kernels compile none of this.)
  const long long brow0 = kMask ? bh * p.bmask_hs + static_cast<long long>(2 * pair) * p.nbt : 0;
  const bool has_row1 = 2 * pair + 1 < p.nbt;
  auto block_on = [&](int t, int j) {  // block (query tile 2 pair + t, key tile j) on?
    return t == 0 ? p.bmask[brow0 + j] != 0 : (has_row1 && p.bmask[brow0 + p.nbt + j] != 0);
  };
  auto next_kv = [&](int j) {  // first visited key tile >= j (jhi + 1 if none)
    if (kMask)
      while (j <= jhi && !block_on(0, j) && !block_on(1, j)) ++j;
    return j;
  };
  // Packed: a unit past its sequence's end has nothing to compute or store (its
  // rows belong to the next sequence): the whole CTA leaves before any setup.
  if (packed && q0 >= Lb) return;
  int nkv = max(0, jhi - jlo + 1);
  if (qlast < q0) nkv = 0;  // the whole pair is padding
  if (kMask && nkv > 0) {
    nkv = 0;
    for (int j = next_kv(jlo); j <= jhi; j = next_kv(j + 1)) ++nkv;
  }

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < C::kStages; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&s_full[t], 1);
      mbar_init(&p_full[t], 128);
      for (int i = 0; i < 3; ++i) mbar_init(&p_part[3 * t + i], 128);
      mbar_init(&o_full[t], 1);
      mbar_init(&epi_bar[t], 128);
    }
    mbar_init(mma_idle, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 8) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (threadIdx.x == 0) {
    FA_TRACE_AT(6, 0, 0);
    uint32_t smid;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
    FA_TRACE_CTA(0, smid);
    FA_TRACE_CTA(1, nkv);
    FA_TRACE_CTA(2, globaltimer_ns());
  }

  if (warp >= 8) {
    regs_dec<72>();
    if (warp == 9 && lane == 0) {
      // ---------------------------------------------------------- producer
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      const bool stall = g_debug_stall != 0;  // test hook: Q never arrives
      if (nkv > 0 && !stall) {
        mbar_arrive_expect_tx(q_full, 2 * C::kTileBytes);
        for (int t = 0; t < 2; ++t)
          for (int c = 0; c < C::kChunks; ++c)
            if constexpr (kStrided)
              tma_load_tile(&tmQ, p.map4 & kMapQ, q_full, sQ + t * C::kTileBytes + c * 16384, c * 64,
                            rb + q0 + t * 128, cbh, h, cb);
            else
              tma_load_3d(&tmQ, q_full, sQ + t * C::kTileBytes + c * 16384, c * 64, q0 + t * 128, bh);
      }
      int issued[C::kStages];
#pragma unroll
      for (int i = 0; i < C::kStages; ++i) issued[i] = 0;
      int it = 0;
      int jcur = next_kv(jlo);
      for (int jj = 0; jj < nkv && !*abort_flag; ++jj, jcur = next_kv(jcur + 1)) {
        const int kv0 = jcur * 128;
        for (int which = 0; which < 2; ++which, ++it) {
          const int s = it % C::kStages;
          if (!mbar_wait(&kv_empty[s], ((it / C::kStages) & 1) ^ 1, abort_flag)) break;
          mbar_arrive_expect_tx(&kv_full[s], C::kTileBytes);
          const CUtensorMap* m = which == 0 ? &tmK : &tmV;
          for (int c = 0; c < C::kChunks; ++c) {
            if constexpr (kStrided)
              tma_load_tile(m, p.map4 & (which == 0 ? kMapK : kMapV), &kv_full[s], sKV + s * C::kTileBytes + c * 16384,
                            c * 64, rb + kv0, ckvh, h / p.g, cb);
            else
              tma_load_3d(m, &kv_full[s], sKV + s * C::kTileBytes + c * 16384, c * 64, kv0, kvh);
          }
          ++issued[s];
        }
      }
      // Never leave the CTA with copies still landing in shared memory.
      if (nkv > 0 && !stall) mbar_wait_drain(q_full, 0);
      for (int s = 0; s < C::kStages; ++s)
        if (issued[s] > 0) mbar_wait_drain(&kv_full[s], (issued[s] - 1) & 1);
    } else if (warp == 8 && lane == 0) {
      // ---------------------------------------------------------- MMA issuer
      const uint32_t aQ = smem_u32(sQ), aKV = smem_u32(sKV);
      constexpr uint32_t kIdescS = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t kIdescO = idesc_bf16_f32(128, D, false, true);
      auto qk = [&](int t, int slot) {  // S_t = Q_t K^T
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t off = (k >> 2) * 16384 + (k & 3) * 32;
          umma_ss(tmem + t * 128, sdesc_sw128(aQ + t * C::kTileBytes + off, 16, 1024),
                  sdesc_sw128(aKV + slot * C::kTileBytes + off, 16, 1024), kIdescS, k > 0);
        }
      };
      // O_t += P_t V, each key range issued once its part of P_t is stored
      // (false: the wait gave up).
      auto pv = [&](int t, int slot, bool acc, uint32_t parity, int tj) {
        constexpr int kStep = 8 / C::kPvParts;
#pragma unroll
        for (int i = 0; i < C::kPvParts; ++i) {
          if (!mbar_wait(i + 1 < C::kPvParts ? &p_part[3 * t + i] : &p_full[t], parity, abort_flag)) return false;
          FA_TRACE_AT(2 + t, tj, i);
          tc_fence_after();
#pragma unroll
          for (int k = i * kStep; k < (i + 1) * kStep; ++k)
            umma_ts(tmem + 256 + t * D, tmem + t * 128 + k * 8,
                    sdesc_sw128(aKV + slot * C::kTileBytes + k * 2048, 16384, 1024), kIdescO, acc || k > 0);
        }
        return true;
      };
      bool ok = nkv > 0 && mbar_wait(q_full, 0, abort_flag);
      // decode: a second query tile of padding rows only gets no products
      bool has1 = true;
      if constexpr (kDecode) has1 = q0 + 128 < Lb;
      int it = 0;
      for (int jj = 0; ok && jj < nkv; ++jj, it += 2) {
        const int sK = it % C::kStages;
        if (!(ok = mbar_wait(&kv_full[sK], (it / C::kStages) & 1, abort_flag))) break;
        FA_TRACE_AT(4, jj, 0);
        tc_fence_after();
        const int sVprev = (it - 1 + C::kStages) % C::kStages;
        if (jj > 0 && !(ok = pv(0, sVprev, jj > 1, (jj - 1) & 1, jj - 1))) break;
        qk(0, sK);
        umma_commit(&s_full[0]);
        if (jj > 0) {
          if (has1 && !(ok = pv(1, sVprev, jj > 1, (jj - 1) & 1, jj - 1))) break;
          umma_commit(&kv_empty[sVprev]);
        }
        if (has1) {
          qk(1, sK);
          umma_commit(&s_full[1]);
        }
        umma_commit(&kv_empty[sK]);
        const int sV = (it + 1) % C::kStages;
        if (!(ok = mbar_wait(&kv_full[sV], ((it + 1) / C::kStages) & 1, abort_flag))) break;
        FA_TRACE_AT(4, jj, 1);
        tc_fence_after();
      }
      if (ok) {
        const int sV = (it - 1) % C::kStages;
        for (int t = 0; t < (has1 ? 2 : 1) && ok; ++t) {
          if (!(ok = pv(t, sV, nkv > 1, (nkv - 1) & 1, nkv - 1))) break;
          umma_commit(&o_full[t]);
        }
      }
      // Before the CTA frees TMEM: every product this thread issued has completed.
      umma_commit(mma_idle);
      mbar_wait_drain(mma_idle, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax (tile t)
    regs_inc<216>();
    const int t = warp >> 2;
    const int wl = warp & 3;
    const int r = wl * 32 + lane;
    const int tq0 = q0 + t * 128;
    const int qrow = tq0 + r;
    const uint32_t lane_off = static_cast<uint32_t>(wl * 32) << 16;
    const uint32_t tS = tmem + lane_off + t * 128;
    const uint32_t tO = tmem + lane_off + 256 + t * D;
    const float sl2 = p.scale_log2;
    float m_used = -INFINITY, l = 0.f, lb = 0.f;
    bool ok = true;
    // positions: of my row, and the smallest / largest of the tile's rows
    int qpos = qrow, tpmin = tq0, tpmax = tq0 + 127;
    if constexpr (kDecode) {
      qpos = qoff + qrow % p.nq;
      decode_positions(tq0, max(tq0, min(tq0 + 127, Lb - 1)), p.nq, qoff, tpmin, tpmax);  // valid rows only
    }
    int nkv_t = nkv;  // key tiles this query tile walks
    if constexpr (kDecode)
      if (t == 1 && q0 + 128 >= Lb) nkv_t = 0;  // padding rows only: no products were issued for them
    int jcur = next_kv(jlo);
    for (int jj = 0; jj < nkv_t; ++jj, jcur = next_kv(jcur + 1)) {
      const int kv0 = jcur * 128;
      // block switched off for this query tile: every score of the tile is masked
      const bool block_off = kMask && !block_on(t, jcur);
      // (warp-uniform outcome: the TMEM loads and stores below are warp-collective)
      ok = mbar_wait(&s_full[t], jj & 1, abort_flag);
      if (!(ok = __all_sync(0xffffffffu, ok))) break;
      if (lane == 0 && wl == 0) FA_TRACE_AT(t, jj, 0);
      tc_fence_after();
      if (kMask && block_off) {  // every weight of the tile is zero: store P = 0 and move on
        uint32_t z[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) z[i] = 0u;
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) tmem_st16(tS + ch * 16, z);
        tmem_wait_st();
        tc_fence_before();
        for (int i = 0; i + 1 < C::kPvParts; ++i) mbar_arrive(&p_part[3 * t + i]);
        mbar_arrive(&p_full[t]);
        continue;
      }
      uint32_t sraw[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tS + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sraw[c * 32]));
      tmem_wait_ld();
      if (lane == 0 && wl == 0) FA_TRACE_AT(t, jj, 2);
      float s[128];
#pragma unroll
      for (int c = 0; c < 128; ++c) s[c] = __uint_as_float(sraw[c]);
      bool full = kv0 + 127 < Lk && !block_off;
      if (p.causal) full = full && (kv0 + 127 <= tpmin);
      if (p.window >= 0) full = full && (tpmax - kv0 <= p.window) && (kv0 + 127 - tpmin <= p.window);
      if (!full) {
        // Tiles on the diagonal / window edge / sequence end only: my row may
        // see key columns [c_lo, c_hi] of the tile; one unsigned compare per element.
        int c_lo = 0, c_hi = block_off ? -1 : min(127, Lk - 1 - kv0);
        if (p.causal) c_hi = min(c_hi, qpos - kv0);
        if (p.window >= 0) {
          c_lo = max(c_lo, qpos - p.window - kv0);
          c_hi = min(c_hi, qpos + p.window - kv0);
        }
        if (c_hi < c_lo) c_lo = 128, c_hi = 128;  // nothing allowed: (c - 128) wraps above the span
        const uint32_t span = static_cast<uint32_t>(c_hi - c_lo);
#pragma unroll
        for (int c = 0; c < 128; ++c) s[c] = static_cast<uint32_t>(c - c_lo) <= span ? s[c] : -INFINITY;
      }
      // Eight independent partial maxima (short dependency chains): mx8[i] covers
      // columns i, i + 8, ..., i + 120.
      float mx8[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) mx8[i] = fmax3(s[i], s[8 + i], s[16 + i]);
#pragma unroll
      for (int c = 24; c < 120; c += 16)
#pragma unroll
        for (int i = 0; i < 8; ++i) mx8[i] = fmax3(mx8[i], s[c + i], s[c + 8 + i]);
#pragma unroll
      for (int i = 0; i < 8; ++i) mx8[i] = fmaxf(mx8[i], s[120 + i]);
      const float mx = fmaxf(fmax3(mx8[0], mx8[1], mx8[2]), fmaxf(fmax3(mx8[3], mx8[4], mx8[5]), fmax3(mx8[6], mx8[7], mx8[7])));
      const float m_new = fmaxf(m_used, mx * sl2);
      bool need = false;
      if (m_used == -INFINITY) {
        m_used = m_new;  // nothing accumulated yet (or only exact zeros)
      } else if (m_new > m_used + kTau) {
        need = true;
      }
      if (__any_sync(0xffffffffu, need)) {
        const float alpha = need ? fast_exp2(m_used - m_new) : 1.f;
        if (need) {
          l *= alpha;
          lb *= alpha;
          m_used = m_new;
        }
#pragma unroll 1
        for (int c = 0; c < D; c += 32) {
          uint32_t o[32];
          tmem_ld32(tO + c, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st32(tO + c, o);
        }
        tmem_wait_st();
      }
      const float ms = (m_used == -INFINITY) ? 0.f : m_used;
      if (lane == 0 && wl == 0) FA_TRACE_AT(t, jj, 3);
      if (full && C::kPolyExp)
        exp_row_to_tmem<true, C::kPvParts>(s, sl2, ms, tS, l, lb, p_part + 3 * t);
      else
        exp_row_to_tmem<false, C::kPvParts>(s, sl2, ms, tS, l, lb, p_part + 3 * t);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&p_full[t]);
      if (lane == 0 && wl == 0) FA_TRACE_AT(t, jj, 1);
    }
    if (kSplit) {
      // ------------------------------------------------ partial results
      const int n = tq0 + r;  // < nq2 always
      const size_t sbh = static_cast<size_t>(split) * BH + bh;
      if (nkv_t <= 0) {
        p.part_m[sbh * p.nq2 + n] = make_float4(-INFINITY, 0.f, 0.f, 0.f);
      } else if (ok && (ok = __all_sync(0xffffffffu, mbar_wait(&o_full[t], 0, abort_flag)))) {
        tc_fence_after();
        float* dst = p.part_o + fwd_part_unit<D>(sbh, p.nq2, n >> 5, 0) + 4 * lane;
#pragma unroll 1
        for (int c = 0; c < D; c += 32) {
          uint32_t o[32];
          tmem_ld32(tO + c, o);  // warp-collective: every lane loads
          tmem_wait_ld();
          if (n < Lb) {  // padding rows get weight 0 in the merge, which never reads their O~
#pragma unroll
            for (int u = 0; u < 8; ++u)
              *reinterpret_cast<uint4*>(dst + 32 * (c + 4 * u)) =
                  make_uint4(o[4 * u], o[4 * u + 1], o[4 * u + 2], o[4 * u + 3]);
          }
        }
        p.part_m[sbh * p.nq2 + n] = n < Lb ? make_float4(m_used, l, lb, 0.f) : make_float4(-INFINITY, 0.f, 0.f, 0.f);
      }
    } else {
    if (ok && nkv > 0) ok = mbar_wait(&o_full[t], 0, abort_flag);
    ok = __all_sync(0xffffffffu, ok);
    if (ok) {
      tc_fence_after();
      const bool pad_row = qrow >= Lb;
      if (pad_row) l = 0.f;
      const float inv = (lb > 0.f && !pad_row) ? 1.f / lb : 0.f;
      uint8_t* sO = sQ + t * C::kTileBytes;  // Q_t is no longer read
      // packed: the sequence ends inside this tile, so each valid row is stored by its own thread
      __nv_bfloat16* orow = nullptr;
      if constexpr (kStrided)
        if (packed && tq0 + 128 > Lb && qrow < Lb)
          orow = static_cast<__nv_bfloat16*>(p.o) + static_cast<long long>(rb + qrow) * p.o_rs +
                 static_cast<long long>(h) * p.o_hs;
#pragma unroll 1
      for (int c = 0; c < D; c += 32) {
        uint32_t o[32];
        if (nkv > 0) {
          tmem_ld32(tO + c, o);
          tmem_wait_ld();
        } else {  // no key tile at all (block mask): O = 0, LSE = -inf
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = 0u;
        }
        const int chunk = c >> 6, u0 = (c & 63) >> 3;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          uint4 val;
          val.x = pack_bf16x2(__uint_as_float(o[8 * u + 0]) * inv, __uint_as_float(o[8 * u + 1]) * inv);
          val.y = pack_bf16x2(__uint_as_float(o[8 * u + 2]) * inv, __uint_as_float(o[8 * u + 3]) * inv);
          val.z = pack_bf16x2(__uint_as_float(o[8 * u + 4]) * inv, __uint_as_float(o[8 * u + 5]) * inv);
          val.w = pack_bf16x2(__uint_as_float(o[8 * u + 6]) * inv, __uint_as_float(o[8 * u + 7]) * inv);
          const uint32_t off = chunk * 16384 + r * 128 + (((u0 + u) ^ (r & 7)) << 4);
          *reinterpret_cast<uint4*>(sO + off) = val;
          if (kStrided && orow) *reinterpret_cast<uint4*>(orow + c + 8 * u) = val;
        }
      }
      const float lse_v = (l > 0.f) ? (m_used + log2f(l)) * kLn2 : -INFINITY;
      if (packed) {
        if (qrow < Lb) p.lse[static_cast<size_t>(rb) * p.H + static_cast<size_t>(h) * Lb + qrow] = lse_v;
      } else if (qrow < p.N) {
        p.lse[static_cast<size_t>(bh) * p.N + qrow] = lse_v;
      }
      fence_proxy_async_smem();
    }
    // Every thread arrives (even after an abort) so the storing thread's
    // bounded wait below cannot be left short of arrivals by a live peer.
    mbar_arrive(&epi_bar[t]);
    // packed: only whole tiles go through the TMA unit (its stores clip at the
    // tensor's end, not at the sequence's)
    const bool tma_out = packed ? tq0 + 128 <= Lb : tq0 < p.N;
    if (ok && r == 0 && tma_out && mbar_wait(&epi_bar[t], 0, abort_flag)) {
      for (int c = 0; c < C::kChunks; ++c) {
        if constexpr (kStrided)
          tma_store_tile(&tmO, p.map4 & kMapO, sQ + t * C::kTileBytes + c * 16384, c * 64, rb + tq0, cbh, h, cb);
        else
          tma_store_3d(&tmO, sQ + t * C::kTileBytes + c * 16384, c * 64, tq0, bh);
      }
      bulk_commit();
      bulk_wait_read0();
    }
    }  // !kSplit
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
  if (threadIdx.x == 0) {
    FA_TRACE_AT(6, 0, 1);
    FA_TRACE_CTA(3, globaltimer_ns());
  }
}

// ---------------------------------------------------------------- split-KV merge
// Merges the per-chunk partial states of each query row with the block-merge
// identity of "Flash attention and efficient attention" (Derivation, Step 3),
// in base 2: m = max_s m_s, w_s = 2^(m_s - m),
//   O = sum_s w_s O~_s / sum_s w_s lb_s,   LSE = (m + log2 sum_s w_s l_s) ln 2.
// One block per (head, 32-row group): eight threads per row compute its
// weights (two chunks each, combined by shuffles), all threads combine the
// 16-byte units (coalesced over rows), and the bf16 rows are written coalesced
// after a transpose through shared memory.
constexpr int kMaxSplits = 16;

template <int D>
__global__ void __launch_bounds__(256) fwd_combine_kernel(const FwdParams p, void* out) {
  __shared__ float wgt[32][kMaxSplits];
  __shared__ float tile[32][D + 4];
  const int groups = (p.N + 31) / 32;
  const int BH = p.B * p.H;
  const size_t bh = blockIdx.x / groups;
  const int g = static_cast<int>(blockIdx.x % groups);
  {  // weights: eight threads per row, each over chunks j and j + 8, combined by shuffles
    const int row = threadIdx.x >> 3, j = threadIdx.x & 7;
    const int n = 32 * g + row;
    float4 st[2];
    float m = -INFINITY;
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int s = j + 8 * k;
      st[k] = s < p.splits ? p.part_m[(static_cast<size_t>(s) * BH + bh) * p.nq2 + n]
                           : make_float4(-INFINITY, 0.f, 0.f, 0.f);
      m = fmaxf(m, st[k].x);
    }
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float w[2], wl = 0.f, wlb = 0.f;
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      w[k] = (st[k].x == -INFINITY) ? 0.f : exp2f(st[k].x - m);
      wl += w[k] * st[k].y;
      wlb += w[k] * st[k].z;
    }
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) {
      wl += __shfl_xor_sync(0xffffffffu, wl, o);
      wlb += __shfl_xor_sync(0xffffffffu, wlb, o);
    }
    const float inv = wlb > 0.f ? 1.f / wlb : 0.f;
#pragma unroll
    for (int k = 0; k < 2; ++k)
      if (j + 8 * k < p.splits) wgt[row][j + 8 * k] = w[k] * inv;
    if (j == 0 && n < p.N) p.lse[bh * p.N + n] = (wl > 0.f) ? (m + log2f(wl)) * kLn2 : -INFINITY;
  }
  __syncthreads();
#pragma unroll
  for (int k = 0; k < D / 32; ++k) {  // 32 rows x D/4 units, 256 threads
    const int f = threadIdx.x + 256 * k;
    const int u = f >> 5, l = f & 31;
    // all chunks' loads issued before the sums (independent, one latency)
    float4 a[kMaxSplits];
    float wv[kMaxSplits];
#pragma unroll
    for (int s = 0; s < kMaxSplits; ++s) {
      wv[s] = s < p.splits ? wgt[l][s] : 0.f;
      a[s] = wv[s] != 0.f  // empty chunk or no allowed key: O~ unused
                 ? *reinterpret_cast<const float4*>(
                       p.part_o + fwd_part_unit<D>(static_cast<size_t>(s) * BH + bh, p.nq2, g, u) + 4 * l)
                 : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int s = 0; s < kMaxSplits; ++s) {
      acc.x = fmaf(wv[s], a[s].x, acc.x);
      acc.y = fmaf(wv[s], a[s].y, acc.y);
      acc.z = fmaf(wv[s], a[s].z, acc.z);
      acc.w = fmaf(wv[s], a[s].w, acc.w);
    }
    *reinterpret_cast<float4*>(&tile[l][4 * u]) = acc;
  }
  __syncthreads();
#pragma unroll
  for (int k = 0; k < D / 32; ++k) {
    const int f = threadIdx.x + 256 * k;
    const int rr = f / (D / 4), u = f % (D / 4);
    const int n = 32 * g + rr;
    if (n >= p.N) continue;
    uint2 v;
    v.x = pack_bf16x2(tile[rr][4 * u + 0], tile[rr][4 * u + 1]);
    v.y = pack_bf16x2(tile[rr][4 * u + 2], tile[rr][4 * u + 3]);
    *reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(out) + (bh * p.N + n) * D + 4 * u) = v;
  }
}

}  // namespace fa
