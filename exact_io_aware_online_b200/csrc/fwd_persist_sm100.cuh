// fwd_persist_sm100.cuh -- persistent bf16 attention forward for short work units.
//
// The same per-tile algorithm and roles as fwd_sm100_kernel (online softmax of
// "Flash attention and efficient attention", section "Derivation: Incremental
// Softmax"; scores in TMEM, P as the TMEM operand of P V), but each CTA runs
// work units (query-tile pairs) one after another instead of one unit per CTA:
//   - the K/V ring and every barrier's phase run on from unit to unit;
//   - the next unit's Q loads as soon as this unit's last Q K^T has read sQ
//     (barrier q_empty), so its first products follow this unit's last P V;
//   - O is staged in a tile of its own (sO, one query tile at a time, handed
//     on between the two query tiles by barriers so_free[t]) since sQ already
//     holds the next unit's Q.
// It pays where units are short (a few key tiles: narrow windows, short or
// packed sequences), whose CTA start, first loads and epilogue would otherwise
// take a large share of the time.  Dense and strided / packed layouts; no
// block mask, split-KV or decode (those keep the one-unit kernel).
#pragma once

#include "fwd_sm100.cuh"

namespace fa {

template <int D>
struct FwdPersistCfg {
  using C = FwdCfg<D>;
  static constexpr int kSmemO = C::kTileBytes;
  static constexpr int kNumBars = C::kNumBars + 3;  // + q_empty, so_free[2]
  static constexpr int kSmemBytes = 1024 + C::kSmemQ + C::kSmemKV + kSmemO + 8 * kNumBars + 16;
  static_assert(kSmemBytes <= 232448, "shared memory per CTA");
  // setmaxnreg split: the unit loop needs more than 72 registers in the
  // producer / MMA warpgroup; the softmax rows fit in 208.
  static constexpr int kRegsSoftmax = 208, kRegsOther = 88;
  static_assert(2 * kRegsSoftmax + kRegsOther == 3 * 168, "the split must use exactly the launch's registers");
};

// Geometry of one work unit (query-tile pair `pair` of head bh), computed by
// every role of the CTA from the unit index alone.
struct FwdUnit {
  int bh, h, kvh, q0, Lb;
  int rb, cb, cbh, ckvh;  // tensor-map coordinates: first row, batch entry, head, kv head
  int jlo, nkv;           // first key tile and the number of key tiles
  bool packed;
  bool skip;  // packed: the unit lies past its sequence's end (its rows belong to the next one)
};

template <bool kStrided>
__device__ __forceinline__ FwdUnit fwd_unit(const FwdArgs<kStrided, false>& p, int unit) {
  FwdUnit U;
  const int BH = p.B * p.H;
  const int per_group = p.group * p.npairs;
  const int grp = unit / per_group;
  const int g0 = grp * p.group;
  const int gsz = min(p.group, BH - g0);
  const int rem = unit - grp * per_group;
  const int pair = p.npairs - 1 - rem / gsz;
  U.bh = g0 + rem % gsz;
  const int b = U.bh / p.H;
  U.h = U.bh % p.H;
  U.kvh = b * p.Hkv + U.h / p.g;
  U.q0 = pair * 256;
  U.Lb = p.seqlens ? max(0, min(p.seqlens[b], p.N)) : p.N;  // valid rows of this batch entry
  U.rb = 0;
  U.cb = b;
  U.cbh = U.bh;
  U.ckvh = U.kvh;
  U.packed = false;
  if constexpr (kStrided) {
    if (p.rowoff) {  // offsets clamped to the tensors' rows whatever they hold
      U.packed = true;
      U.rb = min(max(p.rowoff[b], 0), p.T);
      U.Lb = min(min(max(p.rowoff[b + 1], U.rb), p.T) - U.rb, p.N);
      U.cb = 0;
      U.cbh = U.h;
      U.ckvh = U.h / p.g;
    }
  }
  const int qlast = min(U.q0 + 255, U.Lb - 1);
  int jlo = 0, jhi = p.ntiles_kv - 1;
  jhi = min(jhi, (max(U.Lb, 1) - 1) / 128);  // key tiles holding valid rows
  if (p.causal) jhi = min(jhi, qlast / 128);
  if (p.window >= 0) {
    jlo = max(0, U.q0 - p.window) / 128;
    jhi = min(jhi, (qlast + p.window) / 128);
  }
  U.jlo = jlo;
  U.nkv = qlast < U.q0 ? 0 : max(0, jhi - jlo + 1);  // 0: the whole pair is padding
  U.skip = U.packed && U.q0 >= U.Lb;
  return U;
}

// Launch: min(units, SMs) CTAs of 384 threads, FwdPersistCfg<D>::kSmemBytes of
// dynamic shared memory.  Roles as in fwd_sm100_kernel.
template <int D, bool kStrided>
__global__ void __launch_bounds__(384, 1)
    fwd_persist_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                       const FwdArgs<kStrided, false> p) {
  using C = FwdCfg<D>;
  using PC = FwdPersistCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* base = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  uint8_t* sQ = base;
  uint8_t* sKV = base + C::kSmemQ;
  uint8_t* sO = sKV + C::kSmemKV;  // O staging tile, used by one query tile at a time
  uint64_t* bars = reinterpret_cast<uint64_t*>(sO + PC::kSmemO);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;
  uint64_t* kv_empty = bars + 1 + C::kStages;
  uint64_t* s_full = bars + 1 + 2 * C::kStages;
  uint64_t* p_full = s_full + 2;
  uint64_t* o_full = s_full + 4;
  uint64_t* epi_bar = s_full + 6;   // softmax threads -> storing thread: O tile staged
  uint64_t* mma_idle = s_full + 8;  // every product the MMA thread issued has completed
  uint64_t* p_part = s_full + 9;    // [t * 3 + i]: softmax -> MMA, key range i of P_t stored (i < kPvParts - 1)
  uint64_t* q_empty = s_full + 15;  // MMA -> producer: the unit's last Q K^T has read sQ
  // so_free[t]: the other query tile's storing thread -> tile t's softmax
  // threads: its O store has read sO, so tile t may write its O there.  One
  // barrier per direction, each with one arriving and one waiting tile: a
  // tile cannot reach its next wait before the phase it waits for has begun
  // (a single shared barrier let a tile whose own previous arrival was still
  // pending take the older phase for the one it wanted).
  uint64_t* so_free = s_full + 16;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + PC::kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // Units k * G + i for k = 0, 1, ... (G = gridDim.x), i = blockIdx.x on even
  // passes and G - 1 - blockIdx.x on odd ones: the host orders units heaviest
  // first, so alternating directions spread the work evenly over the CTAs.
  const int nunits = p.B * p.H * p.npairs;
  auto unit_of = [&](int k) -> int {
    const int G = static_cast<int>(gridDim.x);
    const int i = (k & 1) ? G - 1 - static_cast<int>(blockIdx.x) : static_cast<int>(blockIdx.x);
    const int u = k * G + i;
    return u < nunits ? u : -1;
  };

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    mbar_init(&so_free[0], 1);
    mbar_init(&so_free[1], 1);
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

  if (warp >= 8) {
    regs_dec<PC::kRegsOther>();
    if (warp == 9 && lane == 0) {
      // ---------------------------------------------------------- producer
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      const bool stall = g_debug_stall != 0;  // test hook: Q never arrives
      int it = 0;  // K/V loads issued: the ring position, running on from unit to unit
      int uq = 0;  // Q loads issued (one per unit with key tiles)
      for (int k = 0; !*abort_flag; ++k) {
        const int u = unit_of(k);
        if (u < 0) break;
        const FwdUnit U = fwd_unit<kStrided>(p, u);
        if (U.skip || U.nkv == 0) continue;
        if (!stall) {
          // sQ is free once the previous unit's last Q K^T has completed
          if (uq > 0 && !mbar_wait(q_empty, (uq - 1) & 1, abort_flag)) break;
          mbar_arrive_expect_tx(q_full, 2 * C::kTileBytes);
          for (int t = 0; t < 2; ++t)
            for (int c = 0; c < C::kChunks; ++c)
              if constexpr (kStrided)
                tma_load_tile(&tmQ, p.map4 & kMapQ, q_full, sQ + t * C::kTileBytes + c * 16384, c * 64,
                              U.rb + U.q0 + t * 128, U.cbh, U.h, U.cb);
              else
                tma_load_3d(&tmQ, q_full, sQ + t * C::kTileBytes + c * 16384, c * 64, U.q0 + t * 128, U.bh);
          ++uq;
        }
        for (int jj = 0; jj < U.nkv && !*abort_flag; ++jj) {
          const int kv0 = (U.jlo + jj) * 128;
          for (int which = 0; which < 2; ++which, ++it) {
            const int s = it % C::kStages;
            if (!mbar_wait(&kv_empty[s], ((it / C::kStages) & 1) ^ 1, abort_flag)) break;
            mbar_arrive_expect_tx(&kv_full[s], C::kTileBytes);
            const CUtensorMap* m = which == 0 ? &tmK : &tmV;
            for (int c = 0; c < C::kChunks; ++c) {
              if constexpr (kStrided)
                tma_load_tile(m, p.map4 & (which == 0 ? kMapK : kMapV), &kv_full[s],
                              sKV + s * C::kTileBytes + c * 16384, c * 64, U.rb + kv0, U.ckvh, U.h / p.g, U.cb);
              else
                tma_load_3d(m, &kv_full[s], sKV + s * C::kTileBytes + c * 16384, c * 64, kv0, U.kvh);
            }
          }
        }
      }
      // Never leave the CTA with copies still landing in shared memory.
      if (uq > 0) mbar_wait_drain(q_full, (uq - 1) & 1);
      for (int s = 0; s < C::kStages; ++s) {  // loads go round the ring: stage s took this many
        const int issued = it / C::kStages + (s < it % C::kStages ? 1 : 0);
        if (issued > 0) mbar_wait_drain(&kv_full[s], (issued - 1) & 1);
      }
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
      auto pv = [&](int t, int slot, bool acc, uint32_t parity) {
        constexpr int kStep = 8 / C::kPvParts;
#pragma unroll
        for (int i = 0; i < C::kPvParts; ++i) {
          if (!mbar_wait(i + 1 < C::kPvParts ? &p_part[3 * t + i] : &p_full[t], parity, abort_flag)) return false;
          tc_fence_after();
#pragma unroll
          for (int k = i * kStep; k < (i + 1) * kStep; ++k)
            umma_ts(tmem + 256 + t * D, tmem + t * 128 + k * 8,
                    sdesc_sw128(aKV + slot * C::kTileBytes + k * 2048, 16384, 1024), kIdescO, acc || k > 0);
        }
        return true;
      };
      int it = 0;  // K/V ring position, as the producer's
      int um = 0;  // units with key tiles done (q_full parity)
      int kt = 0;  // key tiles done (s_full / P barrier parity)
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int u = unit_of(k);
        if (u < 0) break;
        const FwdUnit U = fwd_unit<kStrided>(p, u);
        if (U.skip || U.nkv == 0) continue;
        const int nkv = U.nkv;
        if (!(ok = mbar_wait(q_full, um & 1, abort_flag))) break;
        for (int jj = 0; jj < nkv; ++jj, it += 2) {
          const int sK = it % C::kStages;
          if (!(ok = mbar_wait(&kv_full[sK], (it / C::kStages) & 1, abort_flag))) break;
          tc_fence_after();
          const int sVprev = (it - 1 + C::kStages) % C::kStages;
          const uint32_t pp = (kt + jj - 1) & 1;  // the previous key tile's P barriers
          if (jj > 0 && !(ok = pv(0, sVprev, jj > 1, pp))) break;
          qk(0, sK);
          umma_commit(&s_full[0]);
          if (jj > 0) {
            if (!(ok = pv(1, sVprev, jj > 1, pp))) break;
            umma_commit(&kv_empty[sVprev]);
          }
          qk(1, sK);
          umma_commit(&s_full[1]);
          if (jj == nkv - 1) umma_commit(q_empty);  // the unit's last read of sQ
          umma_commit(&kv_empty[sK]);
          const int sV = (it + 1) % C::kStages;
          if (!(ok = mbar_wait(&kv_full[sV], ((it + 1) / C::kStages) & 1, abort_flag))) break;
          tc_fence_after();
        }
        if (!ok) break;
        const int sV = (it - 1) % C::kStages;
        const uint32_t pp = (kt + nkv - 1) & 1;
        for (int t = 0; t < 2 && ok; ++t) {
          if (!(ok = pv(t, sV, nkv > 1, pp))) break;
          umma_commit(&o_full[t]);
        }
        if (!ok) break;
        umma_commit(&kv_empty[sV]);  // the unit's last V stage
        kt += nkv;
        ++um;
      }
      // Before the CTA frees TMEM: every product this thread issued has completed.
      umma_commit(mma_idle);
      mbar_wait_drain(mma_idle, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax (tile t)
    regs_inc<PC::kRegsSoftmax>();
    const int t = warp >> 2;
    const int wl = warp & 3;
    const int r = wl * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(wl * 32) << 16;
    const uint32_t tS = tmem + lane_off + t * 128;
    const uint32_t tO = tmem + lane_off + 256 + t * D;
    const float sl2 = p.scale_log2;
    bool ok = true;
    int kt = 0;  // key tiles done (s_full parity)
    int uo = 0;  // units with key tiles done (o_full parity)
    int ne = 0;  // unit epilogues done (epi_bar parity, sO turns)
    for (int k = 0; ok; ++k) {
      const int u = unit_of(k);
      if (u < 0) break;
      const FwdUnit U = fwd_unit<kStrided>(p, u);
      if (U.skip) continue;
      const int tq0 = U.q0 + t * 128;
      const int qrow = tq0 + r;  // my row, also its position
      float m_used = -INFINITY, l = 0.f, lb = 0.f;
      for (int jj = 0; jj < U.nkv; ++jj) {
        const int kv0 = (U.jlo + jj) * 128;
        // (warp-uniform outcome: the TMEM loads and stores below are warp-collective)
        ok = mbar_wait(&s_full[t], (kt + jj) & 1, abort_flag);
        if (!(ok = __all_sync(0xffffffffu, ok))) break;
        tc_fence_after();
        uint32_t sraw[128];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(tS + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sraw[c * 32]));
        tmem_wait_ld();
        float s[128];
#pragma unroll
        for (int c = 0; c < 128; ++c) s[c] = __uint_as_float(sraw[c]);
        bool full = kv0 + 127 < U.Lb;
        if (p.causal) full = full && (kv0 + 127 <= tq0);
        if (p.window >= 0) full = full && (tq0 + 127 - kv0 <= p.window) && (kv0 + 127 - tq0 <= p.window);
        if (!full) {
          // Tiles on the diagonal / window edge / sequence end only: my row may
          // see key columns [c_lo, c_hi] of the tile; one unsigned compare per element.
          int c_lo = 0, c_hi = min(127, U.Lb - 1 - kv0);
          if (p.causal) c_hi = min(c_hi, qrow - kv0);
          if (p.window >= 0) {
            c_lo = max(c_lo, qrow - p.window - kv0);
            c_hi = min(c_hi, qrow + p.window - kv0);
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
        const float mx =
            fmaxf(fmax3(mx8[0], mx8[1], mx8[2]), fmaxf(fmax3(mx8[3], mx8[4], mx8[5]), fmax3(mx8[6], mx8[7], mx8[7])));
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
        if (full && C::kPolyExp)
          exp_row_to_tmem<true, C::kPvParts>(s, sl2, ms, tS, l, lb, p_part + 3 * t);
        else
          exp_row_to_tmem<false, C::kPvParts>(s, sl2, ms, tS, l, lb, p_part + 3 * t);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&p_full[t]);
      }
      if (!ok) break;
      kt += U.nkv;
      // ---------------------------------------------------------- epilogue
      if (U.nkv > 0) ok = mbar_wait(&o_full[t], uo & 1, abort_flag);
      // sO is free once the other query tile's previous store has read it:
      // tile 1 waits for tile 0's store of this unit (so_free[1] completion ne),
      // tile 0 for tile 1's store of the previous unit (so_free[0], ne - 1).
      const int prev = t == 1 ? ne : ne - 1;
      if (ok && prev >= 0) ok = mbar_wait(&so_free[t], prev & 1, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      if (ok) {
        tc_fence_after();
        const bool pad_row = qrow >= U.Lb;
        if (pad_row) l = 0.f;
        const float inv = (lb > 0.f && !pad_row) ? 1.f / lb : 0.f;
        // packed: the sequence ends inside this tile, so each valid row is stored by its own thread
        __nv_bfloat16* orow = nullptr;
        if constexpr (kStrided)
          if (U.packed && tq0 + 128 > U.Lb && qrow < U.Lb)
            orow = static_cast<__nv_bfloat16*>(p.o) + static_cast<long long>(U.rb + qrow) * p.o_rs +
                   static_cast<long long>(U.h) * p.o_hs;
#pragma unroll 1
        for (int c = 0; c < D; c += 32) {
          uint32_t o[32];
          if (U.nkv > 0) {
            tmem_ld32(tO + c, o);
            tmem_wait_ld();
          } else {  // no key tile at all (the pair is padding): O = 0, LSE = -inf
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = 0u;
          }
          const int chunk = c >> 6, u0 = (c & 63) >> 3;
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint4 val;
            val.x = pack_bf16x2(__uint_as_float(o[8 * v + 0]) * inv, __uint_as_float(o[8 * v + 1]) * inv);
            val.y = pack_bf16x2(__uint_as_float(o[8 * v + 2]) * inv, __uint_as_float(o[8 * v + 3]) * inv);
            val.z = pack_bf16x2(__uint_as_float(o[8 * v + 4]) * inv, __uint_as_float(o[8 * v + 5]) * inv);
            val.w = pack_bf16x2(__uint_as_float(o[8 * v + 6]) * inv, __uint_as_float(o[8 * v + 7]) * inv);
            const uint32_t off = chunk * 16384 + r * 128 + (((u0 + v) ^ (r & 7)) << 4);
            *reinterpret_cast<uint4*>(sO + off) = val;
            if (kStrided && orow) *reinterpret_cast<uint4*>(orow + c + 8 * v) = val;
          }
        }
        const float lse_v = (l > 0.f) ? (m_used + log2f(l)) * kLn2 : -INFINITY;
        if (U.packed) {
          if (qrow < U.Lb) p.lse[static_cast<size_t>(U.rb) * p.H + static_cast<size_t>(U.h) * U.Lb + qrow] = lse_v;
        } else if (qrow < p.N) {
          p.lse[static_cast<size_t>(U.bh) * p.N + qrow] = lse_v;
        }
        fence_proxy_async_smem();
      }
      // Every thread arrives (even after an abort) so the storing thread's
      // bounded wait below cannot be left short of arrivals by a live peer.
      mbar_arrive(&epi_bar[t]);
      // packed: only whole tiles go through the TMA unit (its stores clip at the
      // tensor's end, not at the sequence's)
      const bool tma_out = U.packed ? tq0 + 128 <= U.Lb : tq0 < p.N;
      if (r == 0) {
        // Wait for every thread of the tile to have written sO, whether or not
        // it is stored from there: the next wait on epi_bar[t] then finds this
        // phase complete, and sO is released only once nobody writes it.
        const bool staged = mbar_wait(&epi_bar[t], ne & 1, abort_flag);
        if (ok && tma_out && staged) {
          for (int c = 0; c < C::kChunks; ++c) {
            if constexpr (kStrided)
              tma_store_tile(&tmO, p.map4 & kMapO, sO + c * 16384, c * 64, U.rb + tq0, U.cbh, U.h, U.cb);
            else
              tma_store_3d(&tmO, sO + c * 16384, c * 64, tq0, U.bh);
          }
          bulk_commit();
          bulk_wait_read0();
        }
        mbar_arrive(&so_free[1 - t]);  // the other tile may write sO
      }
      if (U.nkv > 0) ++uo;
      ++ne;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

}  // namespace fa
