// Forward attention kernel for sm_100a.
//
// O = softmax(scale * Q K^T [causal]) V and LSE, one head at a time, with the
// online-softmax recurrence over 128-key tiles (marketmaker.cc "The Flash
// Attention algorithm" / "Online softmax recurrence"; ultralytics.com
// glossary "How Flash Attention works").  S and P live only in tensor memory.
//
// Work unit: one (batch*head, pair of 128-row query tiles).  Persistent CTAs
// (one per SM) walk the units with a static stride; causal units are taken
// longest first.  Roles inside a CTA (384 threads = 3 warpgroups):
//   warps 0-3  softmax warpgroup for query tile 0 (thread = row = TMEM lane)
//   warps 4-7  softmax warpgroup for query tile 1
//   warp  8    TMA producer: Q tiles once per unit, K/V tiles through a ring
//   warp  9    MMA issuer (one thread): S_t = Q_t K_j^T and O_t += P_t V_j
//   warps 10-11 idle (they complete the third warpgroup, so that the register
//              split below moves registers within every SM sub-partition)
// Tensor memory (512 columns): S_0 | S_1 | O_0 | O_1.  P (16-bit) is written
// over the first half of its S tile and consumed from there by the PV MMA.
// The two query tiles alternate on the tensor core: while one softmax
// warpgroup exponentiates its S tile, the MMAs of the other tile run.
//
// Rescaling is deferred and conditional: O and l keep a stale running max
// until the max grows by more than 2^8; since O and l are scaled alike, the
// final O / l is unchanged (exactness is kept; only the headroom is bounded).
#include "sm100_ptx.cuh"
#include "fa_kernels.h"

namespace fa {

namespace {

constexpr int kFwdThreads = 384;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale only if max grows > 2^8
// Register split.  Launch: 384 threads x 168 registers.  Warp w runs on SM
// sub-partition w % 4, which therefore holds warps {k, k+4, k+8}: two softmax
// warps and one warp of the producer/MMA warpgroup.  Each sub-partition's
// share after the split must not exceed its launch share (3 x 168).
constexpr int kLaunchRegs = 168;
constexpr int kRegsSoftmax = 216;
constexpr int kRegsOther = 72;
static_assert(2 * kRegsSoftmax + kRegsOther <= 3 * kLaunchRegs, "register split exceeds a sub-partition's pool");

#ifndef FA_FWD_SLOTS_D128
#define FA_FWD_SLOTS_D128 4
#endif

template <int D, bool FP8 = false>
struct FwdLayout {
  static constexpr int kTile = kBlockM * D * (FP8 ? 1 : 2);  // bytes of one 128 x D tile (16- or 8-bit)
  static constexpr int kSlots = (D == 128 && !FP8) ? FA_FWD_SLOTS_D128 : 8;  // K/V ring depth (tiles)
  // Q buffers (each holds the unit's two query tiles).  A second buffer, to
  // prefetch the next unit's Q, measured no faster at d = 64 (the unit
  // boundary is dominated by the causal tile imbalance), so one is used.
  static constexpr int kQBufs = 1;
  static constexpr int kQOff = 0;
  static constexpr int kKVOff = kQBufs * 2 * kTile;
  static constexpr int kBarOff = kKVOff + kSlots * kTile;
  // barrier indices
  static constexpr int kQFull = 0;                  // [kQBufs]
  static constexpr int kQEmpty = kQBufs;            // [kQBufs]
  static constexpr int kKVFull = 2 * kQBufs;
  static constexpr int kKVEmpty = kKVFull + kSlots;
  static constexpr int kSFull = kKVEmpty + kSlots;  // [2]
  static constexpr int kPFull = kSFull + 2;      // [2]
  static constexpr int kOFull = kPFull + 2;      // [2]
  static constexpr int kOEmpty = kOFull + 2;     // [2]
  // Separate P (d = 64, 16-bit): S read by the softmax / P V product done
  static constexpr int kSFree = kOEmpty + 2;     // [2]
  static constexpr int kPVDone = kSFree + 2;     // [2]
  static constexpr int kDrain = kPVDone + 2;
  static constexpr int kNumBars = kDrain + 1;
  // epilogue: per softmax warp a 32-row x 64-byte staging buffer (16-byte
  // chunks XOR-swizzled by row), through which O is stored 8 rows x 64
  // contiguous bytes per store instruction
  static constexpr int kEpiWarpBytes = 32 * 64;
  static constexpr int kEpiOff = (kBarOff + kNumBars * 8 + 127) / 128 * 128;
  static constexpr int kMiscOff = kEpiOff + 8 * kEpiWarpBytes;
  static constexpr int kBytes = kMiscOff + 16;
  static constexpr int kAlloc = kBytes + 1024;  // slack to align the base to 1024 B
  // tensor-memory columns
  static constexpr uint32_t kColS0 = 0;
  static constexpr uint32_t kColO0 = 256;
  static constexpr uint32_t kColP0 = 384;  // separate P (d = 64): P_0 | P_1, 64 columns each
  static_assert(kAlloc <= 232448, "shared memory overflow");
};

struct UnitInfo {
  int bh;    // batch * H + query head
  int kvbh;  // batch * Hkv + key/value head read by that query head
  int r0_0, r0_1;  // first row of query tile 0 / 1
  int nb_0, nb_1;  // key/value tiles each query tile may visit (0 = tile absent)
  int nmax;
  // Key/value tiles actually visited: the union of the two query tiles'
  // active tiles (all of them when dense), K of them; query tile t computes
  // nbk_t of them (dense: its nb_t; block-sparse: the ones it attends).
  int K, nbk_0, nbk_1;
  __device__ __forceinline__ int r0(int t) const { return t ? r0_1 : r0_0; }
  __device__ __forceinline__ int nb(int t) const { return t ? nb_1 : nb_0; }
  __device__ __forceinline__ int nbk(int t) const { return t ? nbk_1 : nbk_0; }
};

// Bits i < 32 of the result: whether row[j0 + i] (a mask byte) is non-zero,
// for j0 + i < n.  The loads are independent, eight in flight at a time (the
// producer and MMA warps run on 72 registers).
__device__ __forceinline__ uint32_t mask_bits(const uint8_t* row, int j0, int n) {
  uint32_t b = 0;
#pragma unroll 8
  for (int i = 0; i < 32; ++i)
    if (j0 + i < n && row[j0 + i] != 0) b |= 1u << i;
  return b;
}

// A 32-block window of a unit's block mask, kept in registers: bit i of w0 /
// w1 says whether query tile 0 / 1 attends key block base + i (always 0 past
// the tile's own nb).  Dense kernels never touch it.
struct MaskWin {
  int base = -32;
  uint32_t w0 = 0, w1 = 0;
  __device__ __forceinline__ void seek(const FwdParams& p, const UnitInfo& ui, int j) {
    if (j >= base && j < base + 32) return;
    base = j & ~31;
    const uint8_t* m = p.bmask + (long long)ui.bh * p.bmask_stride;
    w0 = mask_bits(m + (long long)(ui.r0_0 / kBlockM) * p.n_kv, base, ui.nb_0);
    w1 = ui.nb_1 > 0 ? mask_bits(m + (long long)(ui.r0_1 / kBlockM) * p.n_kv, base, ui.nb_1) : 0u;
  }
  // query tile t attends key block j (j inside the window)
  __device__ __forceinline__ bool tile(int t, int j) const { return ((t ? w1 : w0) >> (j - base)) & 1u; }
};

// Key block j is visited by the unit when either query tile attends it.
template <bool SPARSE>
__device__ __forceinline__ bool unit_block(const FwdParams& p, const UnitInfo& ui, MaskWin& w, int j) {
  if constexpr (!SPARSE) return j < ui.nmax;
  if (j >= ui.nmax) return false;
  w.seek(p, ui, j);
  return ((w.w0 | w.w1) >> (j - w.base)) & 1u;
}

template <bool CAUSAL, bool SPARSE>
__device__ __forceinline__ UnitInfo decode_unit(int u, const FwdParams& p) {
  UnitInfo ui;
  int pair;
  if (CAUSAL) {  // longest units first
    pair = p.n_pairs - 1 - u / p.bh;
    ui.bh = u % p.bh;
  } else {       // neighbouring CTAs share a head (K/V reuse in L2)
    pair = u % p.n_pairs;
    ui.bh = u / p.n_pairs;
  }
  ui.kvbh = (ui.bh / p.H) * (p.H / p.group) + (ui.bh % p.H) / p.group;
  ui.r0_0 = pair * 2 * kBlockM;
  ui.r0_1 = ui.r0_0 + kBlockM;
  ui.nb_0 = CAUSAL ? (ui.r0_0 / kBlockN + 1) : p.n_kv;  // tile 0 always exists
  ui.nb_1 = ui.r0_1 < p.N ? (CAUSAL ? (ui.r0_1 / kBlockN + 1) : p.n_kv) : 0;
  ui.nmax = ui.nb_1 > ui.nb_0 ? ui.nb_1 : ui.nb_0;
  ui.K = ui.nmax;
  ui.nbk_0 = ui.nb_0;
  ui.nbk_1 = ui.nb_1;
  if constexpr (SPARSE) {
    ui.K = ui.nbk_0 = ui.nbk_1 = 0;
    MaskWin w;
    for (int j0 = 0; j0 < ui.nmax; j0 += 32) {
      w.seek(p, ui, j0);
      const uint32_t any = w.w0 | w.w1;
      // visited blocks below each tile's own nb
      ui.K += __popc(any);
      ui.nbk_0 += __popc(w.w0);    // blocks tile 0 attends (w0 is 0 past nb_0)
      ui.nbk_1 += __popc(w.w1);
    }
  }
  return ui;
}

// K-major SW128 operand (Q tile or K tile): rows of 64 elements (128 B);
// a D-wide tile is stored as D/64 column blocks of 128 rows x 128 B.
template <int D>
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t tile, int kstep) {
  const uint32_t addr = tile + (uint32_t)(kstep >> 2) * (kBlockM * 128) + (uint32_t)(kstep & 3) * 32;
  return make_sdesc_sw128(addr, 16, 1024);
}
// Byte offset of K step `kstep` in such a tile (for sdesc_advance).
__host__ __device__ constexpr uint32_t kmajor_off(int kstep) {
  return (uint32_t)(kstep >> 2) * (kBlockM * 128) + (uint32_t)(kstep & 3) * 32;
}

// V tile as the MN-major B operand of O += P V: N = head dim (contiguous),
// K = key index.  Column blocks of 64 are kBlockN*128 bytes apart (LBO),
// 8-key groups 1024 bytes apart (SBO); one 16-key K step = 2048 bytes.
__device__ __forceinline__ uint64_t v_desc(uint32_t tile, int kstep) {
  return make_sdesc_sw128(tile + (uint32_t)kstep * 2048, kBlockN * 128, 1024);
}

// FP8 variant (D = 128): Q, K and V^T arrive as float8 e4m3 codes; the two
// products run as kind::f8f6f4 (K = 32 per instruction: the same 32-byte
// steps through the 128-byte swizzled rows); S is dequantised with the
// product of the Q-block and K-block scales folded into the exponent's
// factor; P is rounded to e4m3 (four per tensor-memory column) for the P V
// product, whose B operand is the transposed V tile (K-major: a row per head
// dimension, 128 keys); the epilogue applies V's per-channel scales.  The
// running sum l adds the unrounded P.  P stays within [0, 2^8] (the stale
// max is at most 2^8 below the true one), inside e4m3's range of 448.
template <int D, bool BF16, bool O32, bool CAUSAL, bool SPARSE, bool FP8 = false, bool SEPP = false>
__global__ void __launch_bounds__(kFwdThreads, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
  static_assert(!FP8 || (D == 128 && !SPARSE), "the FP8 variant is dense, head dim 128");
  using L = FwdLayout<D, FP8>;
  constexpr int kQKBoxes = FP8 ? 1 : D / 64;   // 128-byte column blocks per Q / K tile
  // SEPP (d = 64 leaves 128 tensor-memory columns free): each tile's P gets
  // its own region, so S_t(j+1) can be issued as soon as the softmax has read
  // S_t(j) (instead of after P_t(j) has been consumed) and each tile's
  // softmax runs block after block; the two tiles' softmaxes overlap.  The
  // softmax waits for the previous P V product before it rescales O or
  // overwrites P.  This shortens the per-block chain (a gain for short
  // sequences, whose units are a few blocks long) but makes the softmaxes
  // share the MUFU (a loss on long sequences); the launcher chooses.
  constexpr bool kSepP = SEPP && (D == 64) && !FP8 && !SPARSE;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t bars = base + L::kBarOff;
  auto BAR = [&](int i) -> uint32_t { return bars + 8u * (uint32_t)i; };
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(gbase + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + L::kMiscOff + 4);

  if (threadIdx.x == 0) {
    for (int b = 0; b < L::kQBufs; ++b) {
      mbar_init(BAR(L::kQFull + b), 1);
      mbar_init(BAR(L::kQEmpty + b), 1);
    }
    for (int s = 0; s < L::kSlots; ++s) {
      mbar_init(BAR(L::kKVFull + s), 1);
      mbar_init(BAR(L::kKVEmpty + s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(BAR(L::kSFull + t), 1);
      mbar_init(BAR(L::kPFull + t), 128);
      mbar_init(BAR(L::kOFull + t), 1);
      mbar_init(BAR(L::kOEmpty + t), 128);
      mbar_init(BAR(L::kSFree + t), 128);
      mbar_init(BAR(L::kPVDone + t), 1);
    }
    mbar_init(BAR(L::kDrain), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kProducerWarp) {
    tmem_alloc(smem_u32(const_cast<uint32_t*>(tmem_slot)), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtx wc{p.wait_limit_ns, abort_flag, p.status};
  // nothing above touched global memory: from here on the previous kernel's
  // results are needed (and its reads of O and LSE must be over)
  grid_dependency_wait();
  grid_dependents_launch();

  if (warp >= 8) regs_dec<kRegsOther>();
  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      const uint64_t pol_kv = l2_policy_evict_last();
      const uint64_t pol_q = l2_policy_evict_first();
      uint32_t kv_iter = 0, unit_iter = 0;
      bool ok = true;
      for (int k = 0, u = unit_of(0); u < p.n_units && ok; u = unit_of(++k), ++unit_iter) {
        const UnitInfo ui = decode_unit<CAUSAL, SPARSE>(u, p);
        const uint32_t qb = unit_iter % L::kQBufs, quse = unit_iter / L::kQBufs;
        if (quse > 0 && !mbar_wait(BAR(L::kQEmpty + qb), (quse - 1) & 1, wc)) { ok = false; break; }
        const uint32_t qbytes = (ui.nb_1 > 0 ? 2u : 1u) * L::kTile;
        mbar_arrive_expect_tx(BAR(L::kQFull + qb), qbytes);
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          if (ui.nb(t) == 0) continue;
#pragma unroll
          for (int c = 0; c < kQKBoxes; ++c)
            tma_load_3d(base + L::kQOff + (qb * 2 + t) * L::kTile + c * (kBlockM * 128), &tmQ, BAR(L::kQFull + qb), c * 64,
                        ui.r0(t), ui.bh, pol_q);
        }
        MaskWin mw;
        for (int j = 0; j < ui.nmax && ok; ++j) {
          if (!unit_block<SPARSE>(p, ui, mw, j)) continue;
          for (int kv = 0; kv < 2; ++kv, ++kv_iter) {
            const uint32_t slot = kv_iter % L::kSlots;
            const uint32_t use = kv_iter / L::kSlots;
            if (use > 0 && !mbar_wait(BAR(L::kKVEmpty + slot), (use - 1) & 1, wc)) { ok = false; break; }
            mbar_arrive_expect_tx(BAR(L::kKVFull + slot), L::kTile);
            if (FP8 && kv) {
              // V^T tile: 128 head dims x 128 keys (x = key, y = dim)
              tma_load_3d(base + L::kKVOff + slot * L::kTile, &tmV, BAR(L::kKVFull + slot), j * kBlockN, 0, ui.kvbh,
                          pol_kv);
            } else {
              for (int c = 0; c < kQKBoxes; ++c)
                tma_load_3d(base + L::kKVOff + slot * L::kTile + c * (kBlockN * 128), kv ? &tmV : &tmK,
                            BAR(L::kKVFull + slot), c * 64, j * kBlockN, ui.kvbh, pol_kv);
            }
          }
        }
      }
      if (!ok) {
        // Let every copy already issued land before the CTA exits.
        for (uint32_t s = 0; s < (uint32_t)L::kSlots; ++s) {
          const uint32_t issued = kv_iter / L::kSlots + (s < kv_iter % L::kSlots ? 1u : 0u);
          if (issued > 0) mbar_wait_drain(BAR(L::kKVFull + s), (issued - 1) & 1, p.wait_limit_ns);
        }
        // unit_iter Q loads were issued (the aborted unit's included or not,
        // both cases leave unit_iter equal to the number issued)
        for (uint32_t b = 0; b < (uint32_t)L::kQBufs; ++b) {
          const uint32_t issued = unit_iter / L::kQBufs + (b < unit_iter % L::kQBufs ? 1u : 0u);
          if (issued > 0) mbar_wait_drain(BAR(L::kQFull + b), (issued - 1) & 1, p.wait_limit_ns);
        }
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      // kind::f8f6f4 with e4m3 operands uses the same fields (format code 0)
      constexpr uint32_t idesc_s = make_idesc_f16(FP8 ? false : BF16, kBlockM, kBlockN, false, false);
      constexpr uint32_t idesc_pv = make_idesc_f16(FP8 ? false : BF16, kBlockM, D, false, !FP8);
      uint32_t kv_iter = 0, unit_iter = 0;
      uint32_t p_cnt0 = 0, p_cnt1 = 0, o_uses0 = 0, o_uses1 = 0;
      uint32_t s_iss0 = 0, s_iss1 = 0;   // S MMAs issued per tile (separate-P pipeline)
      bool ok = true;
      for (int k = 0, u = unit_of(0); u < p.n_units && ok; u = unit_of(++k), ++unit_iter) {
        const UnitInfo ui = decode_unit<CAUSAL, SPARSE>(u, p);
        const uint32_t qb = unit_iter % L::kQBufs;
        if (!mbar_wait(BAR(L::kQFull + qb), (unit_iter / L::kQBufs) & 1, wc)) { ok = false; break; }
        tc_fence_after();
        const uint32_t kv_base = kv_iter;
        if (ui.K == 0) tc_commit(BAR(L::kQEmpty + qb));  // no key block: Q is not read
        if constexpr (kSepP) {
          // Per visited block j: first S_t(j) for both tiles (each after the
          // softmax has read S_t(j-1)), then P_t(j-1) V_{j-1}.
          for (int j = 0; j <= ui.K && ok; ++j) {
            const uint32_t k_idx = kv_base + 2 * j, v_idx = kv_base + 2 * (j - 1) + 1;
            bool k_ready = false, v_ready = false;
#pragma unroll
            for (int t = 0; t < 2; ++t) {
              if (!ok || j >= ui.nb(t)) continue;
              uint32_t& sc = t ? s_iss1 : s_iss0;
              if (sc > 0) ok = mbar_wait(BAR(L::kSFree + t), (sc - 1) & 1, wc);
              if (ok && !k_ready) {
                ok = mbar_wait(BAR(L::kKVFull + k_idx % L::kSlots), (k_idx / L::kSlots) & 1, wc);
                k_ready = true;
              }
              if (!ok) continue;
              tc_fence_after();
              const uint32_t qt = base + L::kQOff + (qb * 2 + t) * L::kTile;
              const uint32_t kt = base + L::kKVOff + (k_idx % L::kSlots) * L::kTile;
              const uint64_t qd = kmajor_desc<D>(qt, 0), kd = kmajor_desc<D>(kt, 0);
#pragma unroll
              for (int ks = 0; ks < D / 16; ++ks)
                mma_ss(tmem + L::kColS0 + 128u * t, sdesc_advance(qd, kmajor_off(ks)), sdesc_advance(kd, kmajor_off(ks)),
                       idesc_s, ks > 0 ? 1u : 0u);
              tc_commit(BAR(L::kSFull + t));
              ++sc;
            }
            if (!ok) break;
#pragma unroll
            for (int t = 0; t < 2; ++t) {
              const int nbt = ui.nb(t);
              if (!ok || j < 1 || j > nbt) continue;
              const uint32_t pc = t ? p_cnt1 : p_cnt0;
              const uint32_t ou = t ? o_uses1 : o_uses0;
              ok = mbar_wait(BAR(L::kPFull + t), pc & 1, wc);
              if (t) ++p_cnt1; else ++p_cnt0;
              if (ok && j == 1 && ou > 0) ok = mbar_wait(BAR(L::kOEmpty + t), (ou - 1) & 1, wc);
              if (ok && !v_ready) {
                ok = mbar_wait(BAR(L::kKVFull + v_idx % L::kSlots), (v_idx / L::kSlots) & 1, wc);
                v_ready = true;
              }
              if (!ok) continue;
              tc_fence_after();
              const uint64_t vd = v_desc(base + L::kKVOff + (v_idx % L::kSlots) * L::kTile, 0);
#pragma unroll
              for (int ks = 0; ks < kBlockN / 16; ++ks)
                mma_ts(tmem + L::kColO0 + (uint32_t)D * t, tmem + L::kColP0 + 64u * t + 8u * ks,
                       sdesc_advance(vd, (uint32_t)ks * 2048), idesc_pv, (j > 1 || ks > 0) ? 1u : 0u);
              tc_commit(BAR(L::kPVDone + t));
              if (j == nbt) tc_commit(BAR(L::kOFull + t));
            }
            if (!ok) break;
            if (j == ui.K - 1) tc_commit(BAR(L::kQEmpty + qb));
            if (j < ui.K) tc_commit(BAR(L::kKVEmpty + k_idx % L::kSlots));
            if (j >= 1) tc_commit(BAR(L::kKVEmpty + v_idx % L::kSlots));
          }
          kv_iter = kv_base + 2 * ui.K;
          o_uses0 += ui.nbk_0 > 0 ? 1u : 0u;
          o_uses1 += ui.nbk_1 > 0 ? 1u : 0u;
          continue;
        }
        // Block-sparse: each query tile computes only the visited blocks it
        // attends (live); the other tile's blocks cost it no MMA and no
        // softmax.  Dense: tile t is live at visited block j iff j < nb_t.
        MaskWin mw;
        int jb_cur = -1;                    // block index of visited block j
        bool live_prev0 = false, live_prev1 = false, live_cur0 = false, live_cur1 = false;
        int pv_done0 = 0, pv_done1 = 0;     // P V products issued per tile
        for (int j = 0; j <= ui.K && ok; ++j) {          // j counts visited blocks
          const uint32_t k_idx = kv_base + 2 * j, v_idx = kv_base + 2 * (j - 1) + 1;
          bool v_ready = false, k_ready = false;
          if constexpr (SPARSE) {
            live_prev0 = live_cur0;
            live_prev1 = live_cur1;
            live_cur0 = live_cur1 = false;
            if (j < ui.K) {
              do { ++jb_cur; } while (!unit_block<SPARSE>(p, ui, mw, jb_cur));
              live_cur0 = mw.tile(0, jb_cur);
              live_cur1 = mw.tile(1, jb_cur);
            }
          }
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            const int nbt = ui.nbk(t);
            if (!ok || nbt == 0) continue;
            const uint32_t colS = L::kColS0 + 128u * t;
            const uint32_t colO = L::kColO0 + (uint32_t)D * t;
            const uint32_t pc = t ? p_cnt1 : p_cnt0;
            const uint32_t ou = t ? o_uses1 : o_uses0;
            bool pv_now, s_now, first, last;
            if constexpr (SPARSE) {
              const int pvd = t ? pv_done1 : pv_done0;
              pv_now = t ? live_prev1 : live_prev0;
              s_now = t ? live_cur1 : live_cur0;
              first = pvd == 0;
              last = pvd + 1 == nbt;
            } else {
              pv_now = j >= 1 && j <= nbt;
              s_now = j < nbt;
              first = j == 1;
              last = j == nbt;
            }
            if (pv_now) {
              // O_t (+)= P_t V_{j-1}
              if constexpr (SPARSE) {
                if (t) ++pv_done1; else ++pv_done0;
              }
              ok = mbar_wait(BAR(L::kPFull + t), pc & 1, wc);
              if (t) ++p_cnt1; else ++p_cnt0;
              if (ok && first && ou > 0) ok = mbar_wait(BAR(L::kOEmpty + t), (ou - 1) & 1, wc);
              if (ok && !v_ready) {
                ok = mbar_wait(BAR(L::kKVFull + v_idx % L::kSlots), (v_idx / L::kSlots) & 1, wc);
                v_ready = true;
              }
              if (!ok) continue;
              tc_fence_after();
              const uint32_t vt = base + L::kKVOff + (v_idx % L::kSlots) * L::kTile;
              // descriptors built once per tile, stepped by constant offsets
              if constexpr (FP8) {
                const uint64_t vd = kmajor_desc<128>(vt, 0);
#pragma unroll
                for (int ks = 0; ks < kBlockN / 32; ++ks)
                  mma_ts_f8(tmem + colO, tmem + colS + 8u * ks, sdesc_advance(vd, kmajor_off(ks)), idesc_pv,
                            (!first || ks > 0) ? 1u : 0u);
              } else {
                const uint64_t vd = v_desc(vt, 0);
#pragma unroll
                for (int ks = 0; ks < kBlockN / 16; ++ks)
                  mma_ts(tmem + colO, tmem + colS + 8u * ks, sdesc_advance(vd, (uint32_t)ks * 2048), idesc_pv,
                         (!first || ks > 0) ? 1u : 0u);
              }
              if (last) tc_commit(BAR(L::kOFull + t));
            }
            if (s_now) {
              // K_j is waited for only here, after the PV MMAs of block j-1
              // (which do not need it) have been issued.
              if (!k_ready) {
                ok = mbar_wait(BAR(L::kKVFull + k_idx % L::kSlots), (k_idx / L::kSlots) & 1, wc);
                k_ready = true;
                if (!ok) continue;
                tc_fence_after();
              }
              // S_t = Q_t K_j^T
              const uint32_t qt = base + L::kQOff + (qb * 2 + t) * L::kTile;
              const uint32_t kt = base + L::kKVOff + (k_idx % L::kSlots) * L::kTile;
              const uint64_t qd = kmajor_desc<D>(qt, 0), kd = kmajor_desc<D>(kt, 0);
              if constexpr (FP8) {
#pragma unroll
                for (int ks = 0; ks < D / 32; ++ks)
                  mma_ss_f8(tmem + colS, sdesc_advance(qd, kmajor_off(ks)), sdesc_advance(kd, kmajor_off(ks)),
                            idesc_s, ks > 0 ? 1u : 0u);
              } else {
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks)
                  mma_ss(tmem + colS, sdesc_advance(qd, kmajor_off(ks)), sdesc_advance(kd, kmajor_off(ks)), idesc_s,
                         ks > 0 ? 1u : 0u);
              }
              tc_commit(BAR(L::kSFull + t));
            }
          }
          if (!ok) break;
          if (j == ui.K - 1) tc_commit(BAR(L::kQEmpty + qb));
          // Release K_j as soon as the S MMAs of block j are issued (they are
          // its last readers) and V_{j-1} after the PV MMAs of block j-1; the
          // producer can then refill the slots about one block ahead.
          if (j < ui.K) tc_commit(BAR(L::kKVEmpty + k_idx % L::kSlots));
          if (j >= 1) tc_commit(BAR(L::kKVEmpty + v_idx % L::kSlots));
        }
        kv_iter = kv_base + 2 * ui.K;
        o_uses0 += ui.nbk_0 > 0 ? 1u : 0u;
        o_uses1 += ui.nbk_1 > 0 ? 1u : 0u;
      }
      // Make sure no MMA is still reading shared memory or writing tensor
      // memory when the CTA leaves (normal exit: they are all done already).
      tc_commit(BAR(L::kDrain));
      mbar_wait_drain(BAR(L::kDrain), 0, p.wait_limit_ns);
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------ softmax
    regs_inc<kRegsSoftmax>();
    const int t = warp >> 2;                       // query tile of this warpgroup
    const int r_in = threadIdx.x & 127;            // row within the tile = TMEM lane
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_off + L::kColS0 + 128u * t;
    const uint32_t tO = tmem + lane_off + L::kColO0 + (uint32_t)D * t;
    const uint32_t tP = kSepP ? tmem + lane_off + L::kColP0 + 64u * t : tS;   // where P goes
    const float sl2 = p.scale_log2;
    uint32_t s_cnt = 0, o_cnt = 0;
    uint32_t p_stored = 0;   // P tiles written (separate-P pipeline: one P V product each)
    int unit_iter = 0;
    bool ok = true;
    for (int k = 0, u = unit_of(0); u < p.n_units && ok; u = unit_of(++k), ++unit_iter) {
      const UnitInfo ui = decode_unit<CAUSAL, SPARSE>(u, p);
      if (ui.nb(t) == 0) continue;                 // query tile past the sequence end
      const int nb = ui.nbk(t);                    // key blocks this tile visits
      const int row = ui.r0(t) + r_in;
      const int qblk = ui.r0(t) / kBlockM;
      // FP8: the query block's dequantisation scale, folded into the factor
      float sq_l2 = sl2;
      if constexpr (FP8) sq_l2 = sl2 * p.fp8_sq[(size_t)ui.bh * p.n_kv + qblk];
      float m_run = -INFINITY, l_run = 0.f;        // m_run stays -inf until a key is seen
      int jb = -1;                                 // index of the current key block
      MaskWin mw;
      for (int j = 0; j < nb; ++j) {
        if constexpr (SPARSE) {
          do { ++jb; } while (!(unit_block<SPARSE>(p, ui, mw, jb) && mw.tile(t, jb)));
        } else {
          ++jb;
        }
        ok = warp_all(mbar_wait(BAR(L::kSFull + t), s_cnt & 1, wc));
        if (!ok) break;
        ++s_cnt;
        tc_fence_after();
        uint32_t sr[kBlockN];
#pragma unroll
        for (int c = 0; c < kBlockN / 32; ++c) tmem_ld32(tS + 32u * c, sr + 32 * c);
        tmem_wait_ld();
        bool pv_seen = false;   // the previous P V product of this tile is known complete
        if constexpr (kSepP) {
          // S_t(j) is in registers: the MMA issuer may overwrite it with S_t(j+1)
          tc_fence_before();
          mbar_arrive(BAR(L::kSFree + t));
        }
        float s[kBlockN];
#pragma unroll
        for (int c = 0; c < kBlockN; ++c) s[c] = __uint_as_float(sr[c]);
        const int kbase = jb * kBlockN;
        // factor from raw scores to log2 units (FP8: times both block scales)
        float c_l2 = sl2;
        if constexpr (FP8) c_l2 = sq_l2 * p.fp8_sk[(size_t)ui.kvbh * p.n_kv + jb];
        if (CAUSAL && jb == qblk) {
#pragma unroll
          for (int c = 0; c < kBlockN; ++c)
            if (kbase + c > row) s[c] = -INFINITY;
        } else if (!CAUSAL && kbase + kBlockN > p.N) {
#pragma unroll
          for (int c = 0; c < kBlockN; ++c)
            if (kbase + c >= p.N) s[c] = -INFINITY;
        }
        // row max: eight independent partial maxima, three inputs per step
        float pm[8];
#pragma unroll
        for (int a = 0; a < 8; ++a) pm[a] = fmaxf(s[a], s[a + 8]);
#pragma unroll
        for (int c = 16; c + 16 <= kBlockN; c += 16)
#pragma unroll
          for (int a = 0; a < 8; ++a) pm[a] = fmax3(pm[a], s[c + a], s[c + a + 8]);
        const float mx = fmax3(fmax3(pm[0], pm[1], pm[2]), fmax3(pm[3], pm[4], pm[5]), fmaxf(pm[6], pm[7]));
        const float m_new = fmaxf(m_run, mx * c_l2);
        // Until a row has seen a key, its O and l are zero: the first finite
        // max is taken as is, without a rescale.
        const bool fresh = m_run == -INFINITY;
        const bool need = !fresh && m_new > m_run + kRescaleThreshold;
        if (fresh) m_run = m_new;
        {
          // The rescale touches tensor memory with warp-collective
          // instructions, so the whole warp takes the branch when any of its
          // rows needs it; rows that do not keep their max and use alpha = 1.
          if (__any_sync(0xffffffffu, need)) {
            if constexpr (kSepP) {
              // O must hold the previous P V product before it is rescaled
              if (p_stored > 0) {
                ok = warp_all(mbar_wait(BAR(L::kPVDone + t), (p_stored - 1) & 1, wc));
                if (!ok) break;
                tc_fence_after();
              }
              pv_seen = true;
            }
            const float alpha = need ? ex2_approx(m_run - m_new) : 1.f;
            if (need) {
              l_run *= alpha;
              m_run = m_new;
            }
            // O_t was last written by PV of tile j-1, which completed before
            // S_j was signalled (tcgen05 ops of one thread complete in order).
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
              uint32_t o[32];
              tmem_ld32(tO + 32u * c, o);
              tmem_wait_ld();
              const uint64_t a2 = f2_pack(alpha, alpha);
#pragma unroll
              for (int e = 0; e < 16; ++e) {
                float lo, hi;
                f2_unpack(f2_mul(f2_pack(__uint_as_float(o[2 * e]), __uint_as_float(o[2 * e + 1])), a2), lo, hi);
                o[2 * e] = __float_as_uint(lo);
                o[2 * e + 1] = __float_as_uint(hi);
              }
              tmem_st32(tO + 32u * c, o);
            }
          }
        }
        const float neg_m = (m_run == -INFINITY) ? 0.f : -m_run;  // -inf row: every P is 0
        // exponents and row sums of key pairs with the two-wide fp32
        // instructions: four pair accumulators (eight partial sums)
        const uint64_t cl2x2 = f2_pack(c_l2, c_l2), nm2 = f2_pack(neg_m, neg_m);
        uint64_t ps2[4] = {0ull, 0ull, 0ull, 0ull};
        uint32_t pk_all[kSepP ? kBlockN / 2 : 1];   // separate P: stored after the wait below
#pragma unroll
        for (int q = 0; q < kBlockN / 32; ++q) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            float x0, x1;
            f2_unpack(f2_fma(f2_pack(s[32 * q + 2 * e], s[32 * q + 2 * e + 1]), cl2x2, nm2), x0, x1);
            const float p0 = ex2_approx(x0);
            const float p1 = ex2_approx(x1);
            ps2[e & 3] = f2_add(ps2[e & 3], f2_pack(p0, p1));
            if constexpr (FP8) {
              // two e4m3 per 16 bits; element pairs (2e, 2e + 1) of 32 keys
              const uint32_t h = pack_e4m3x2(p0, p1);
              if (e & 1) pk[e >> 1] |= h << 16; else pk[e >> 1] = h;
            } else {
              pk[e] = pack2<BF16>(p0, p1);
            }
          }
          if constexpr (kSepP) {
#pragma unroll
            for (int e = 0; e < 16; ++e) pk_all[16 * q + e] = pk[e];
          } else if constexpr (FP8) {
            tmem_st8(tS + 8u * q, pk);   // 32 keys = 8 columns of four e4m3
          } else {
            tmem_st16(tS + 16u * q, pk);
          }
        }
        if constexpr (kSepP) {
          // the previous P of this tile must have been read by its P V product
          if (p_stored > 0 && !pv_seen) {
            ok = warp_all(mbar_wait(BAR(L::kPVDone + t), (p_stored - 1) & 1, wc));
            if (!ok) break;
            tc_fence_after();
          }
#pragma unroll
          for (int q = 0; q < kBlockN / 32; ++q) tmem_st16(tP + 16u * q, pk_all + 16 * q);
          ++p_stored;
        }
        {
          float a0, a1, b0, b1;
          f2_unpack(f2_add(ps2[0], ps2[1]), a0, a1);
          f2_unpack(f2_add(ps2[2], ps2[3]), b0, b1);
          l_run += (a0 + b0) + (a1 + b1);
        }
        tmem_wait_st();
        tc_fence_before();
        const bool withhold = (p.debug_flags & 1) && unit_iter == 0 && j == 0 && t == 0;
        if (!withhold) mbar_arrive(BAR(L::kPFull + t));
      }
      if (!ok) break;
      // ---- epilogue: O / l -> dtype -> global; LSE = (m + log2 l) ln 2.
      // O is read from tensor memory 32 columns at a time, normalised,
      // converted and stored through this warp's staging buffer, so that
      // each store instruction writes 64 contiguous bytes of 8 rows (not 16
      // bytes of 32 rows).  A row with no kept key (block-sparse) gets O = 0
      // and LSE = -inf; a tile that visits no key block at all skips tensor
      // memory entirely.
      if (nb > 0) {
        ok = warp_all(mbar_wait(BAR(L::kOFull + t), o_cnt & 1, wc));
        if (!ok) break;
        ++o_cnt;
        tc_fence_after();
      }
      const float inv_l = l_run > 0.f ? 1.f / l_run : 0.f;
      {
        constexpr int kOBytes = O32 ? 4 : 2;
        constexpr int kGroups = O32 ? 2 : 1;        // 64-byte groups per 32 columns
        const int lane = threadIdx.x & 31;
        uint8_t* stg = gbase + L::kEpiOff + warp * L::kEpiWarpBytes;
        const int row0 = ui.r0(t) + (r_in & ~31);   // first row of this warp's 32
        uint8_t* obase = reinterpret_cast<uint8_t*>(p.o) + (size_t)ui.bh * p.N * D * kOBytes;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          if (nb > 0) {
            tmem_ld32(tO + 32u * c, o);
            tmem_wait_ld();
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = 0u;
          }
          if constexpr (FP8) {  // V's per-channel dequantisation scales
            const float* svp = p.fp8_sv + (size_t)ui.kvbh * D + 32 * c;
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * svp[e]);
          }
#pragma unroll
          for (int gi = 0; gi < kGroups; ++gi) {
            uint32_t w[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              if constexpr (O32) w[e] = __float_as_uint(__uint_as_float(o[16 * gi + e]) * inv_l);
              else w[e] = pack2<BF16>(__uint_as_float(o[2 * e]) * inv_l, __uint_as_float(o[2 * e + 1]) * inv_l);
            }
            // this row's 64 bytes -> row `lane` of the staging buffer, chunk k
            // at position k ^ ((row >> 1) & 3): the row-wise writes and the
            // 8-rows x 4-chunks reads below are both free of bank conflicts
            __syncwarp();
#pragma unroll
            for (int kc = 0; kc < 4; ++kc)
              *reinterpret_cast<uint4*>(stg + lane * 64 + ((kc ^ ((lane >> 1) & 3)) * 16)) =
                  make_uint4(w[4 * kc], w[4 * kc + 1], w[4 * kc + 2], w[4 * kc + 3]);
            __syncwarp();
            const int colb = (c * kGroups + gi) * 64;   // byte offset of the group within a row
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int rr = (lane >> 2) + 8 * i, kc = lane & 3;
              const uint4 val = *reinterpret_cast<const uint4*>(stg + rr * 64 + ((kc ^ ((rr >> 1) & 3)) * 16));
              if (row0 + rr < p.N)
                *reinterpret_cast<uint4*>(obase + (size_t)(row0 + rr) * D * kOBytes + colb + kc * 16) = val;
            }
          }
        }
      }
      if (nb > 0) {
        tc_fence_before();
        mbar_arrive(BAR(L::kOEmpty + t));
      }
      if (row < p.N)
        p.lse[(size_t)ui.bh * p.N + row] = l_run > 0.f ? (m_run + __log2f(l_run)) * 0.69314718055994531f : -INFINITY;
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == kProducerWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int D, bool BF16, bool O32, bool CAUSAL, bool SPARSE, bool SEPP = false>
cudaError_t launch_fwd_t(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                         const FwdParams& p, int grid, cudaStream_t st) {
  auto kern = fa_fwd_kernel<D, BF16, O32, CAUSAL, SPARSE, false, SEPP>;
  constexpr int smem = FwdLayout<D>::kAlloc;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  e = launch_chained(kern, dim3(grid), dim3(kFwdThreads), smem, st, tq, tk, tv, p);
  return e != cudaSuccess ? e : cudaGetLastError();
}

template <int D, bool BF16, bool O32>
cudaError_t launch_fwd_c(bool causal, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                         const FwdParams& p, int grid, cudaStream_t st) {
  const bool sparse = p.bmask != nullptr;
  // separate-P pipeline for short sequences at d = 64 (units of at most 16
  // key blocks): measured faster at N = 1024, slower at N >= 4096
  if constexpr (D == 64) {
    if (!sparse && p.N <= 2048)
      return causal ? launch_fwd_t<D, BF16, O32, true, false, true>(tq, tk, tv, p, grid, st)
                    : launch_fwd_t<D, BF16, O32, false, false, true>(tq, tk, tv, p, grid, st);
  }
  if (causal) return sparse ? launch_fwd_t<D, BF16, O32, true, true>(tq, tk, tv, p, grid, st)
                            : launch_fwd_t<D, BF16, O32, true, false>(tq, tk, tv, p, grid, st);
  return sparse ? launch_fwd_t<D, BF16, O32, false, true>(tq, tk, tv, p, grid, st)
                : launch_fwd_t<D, BF16, O32, false, false>(tq, tk, tv, p, grid, st);
}

template <int D>
cudaError_t launch_fwd_d(bool bf16, bool o32, bool causal, const CUtensorMap& tq, const CUtensorMap& tk,
                         const CUtensorMap& tv, const FwdParams& p, int grid, cudaStream_t st) {
  if (bf16) return o32 ? launch_fwd_c<D, true, true>(causal, tq, tk, tv, p, grid, st)
                       : launch_fwd_c<D, true, false>(causal, tq, tk, tv, p, grid, st);
  return o32 ? launch_fwd_c<D, false, true>(causal, tq, tk, tv, p, grid, st)
             : launch_fwd_c<D, false, false>(causal, tq, tk, tv, p, grid, st);
}

}  // namespace

template <bool BF16, bool O32, bool CAUSAL>
cudaError_t launch_fwd_fp8_t(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tvt,
                             const FwdParams& p, int grid, cudaStream_t st) {
  auto kern = fa_fwd_kernel<128, BF16, O32, CAUSAL, false, true>;
  constexpr int smem = FwdLayout<128, true>::kAlloc;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  kern<<<grid, kFwdThreads, smem, st>>>(tq, tk, tvt, p);
  return cudaGetLastError();
}

int fwd_threads() { return kFwdThreads; }
int fwd_fp8_smem() { return FwdLayout<128, true>::kAlloc; }

cudaError_t launch_fwd_fp8(bool bf16, bool o32, bool causal, const CUtensorMap& tq, const CUtensorMap& tk,
                           const CUtensorMap& tvt, const FwdParams& p, int grid, cudaStream_t st) {
  if (bf16) {
    if (o32) return causal ? launch_fwd_fp8_t<true, true, true>(tq, tk, tvt, p, grid, st)
                           : launch_fwd_fp8_t<true, true, false>(tq, tk, tvt, p, grid, st);
    return causal ? launch_fwd_fp8_t<true, false, true>(tq, tk, tvt, p, grid, st)
                  : launch_fwd_fp8_t<true, false, false>(tq, tk, tvt, p, grid, st);
  }
  if (o32) return causal ? launch_fwd_fp8_t<false, true, true>(tq, tk, tvt, p, grid, st)
                         : launch_fwd_fp8_t<false, true, false>(tq, tk, tvt, p, grid, st);
  return causal ? launch_fwd_fp8_t<false, false, true>(tq, tk, tvt, p, grid, st)
                : launch_fwd_fp8_t<false, false, false>(tq, tk, tvt, p, grid, st);
}

cudaError_t launch_fwd(int d, bool bf16, bool o32, bool causal, const CUtensorMap& tq, const CUtensorMap& tk,
                       const CUtensorMap& tv, const FwdParams& p, int grid, cudaStream_t st) {
  if (d == 64) return launch_fwd_d<64>(bf16, o32, causal, tq, tk, tv, p, grid, st);
  if (d == 128) return launch_fwd_d<128>(bf16, o32, causal, tq, tk, tv, p, grid, st);
  return cudaErrorInvalidValue;
}

}  // namespace fa
