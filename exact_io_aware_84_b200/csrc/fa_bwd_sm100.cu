// Backward attention kernels for sm_100a.
//
// The backward recomputes P from Q, K and the forward's log-sum-exp instead
// of storing it (marketmaker.cc "Backward pass: recompute instead of store").
// With dP = dO V^T, D_i = sum_c dO_ic O_ic and dS = P o (dP - D):
//   dV = P^T dO,  dK = scale dS^T Q,  dQ = scale dS K.
// Three launches:
//   1. fa_bwd_prep:   D_i, -LSE_i * log2(e) (-inf on padding rows), zero dQacc.
//   2. fa_bwd_main:   one CTA per (batch*head, 128-key tile) unit, persistent;
//                     loops over query tiles, keeps dK and dV in tensor memory,
//                     adds each query tile's dQ into the fp32 accumulator with a
//                     bulk shared->global reduce.
//   3. fa_bwd_dq:     dQ = dtype(scale * dQacc).
//
// fa_bwd_main works transposed (keys on the 128 tensor-memory lanes):
//   S^T = K_j Q_i^T, dP^T = V_j dO_i^T            (SS MMAs, M = 128 keys)
//   P^T = exp2(S^T * scale*log2e - LSE_i*log2e)    (compute warpgroups)
//   dS^T = P^T o (dP^T - D_i)                      (compute warpgroups)
//   dV += P^T dO_i, dK += dS^T Q_i                 (TS MMAs, A from TMEM)
//   d = 64 : dQ_i   = dS K_j      (M = 128 queries, both operands MN-major)
//   d = 128: dQ_i^T = K_j^T dS^T  (M = 128 head dims, both operands MN-major)
// Query tile BR = 128 rows for d = 64 and 64 rows for d = 128, so that
// S^T | dP^T | dV | dK | dQ fit in the 512 tensor-memory columns (448 used).
// Roles (512 threads):
//   warps 0-7   two compute warpgroups (thread = key = TMEM lane), each owning
//               half of every query tile's columns: P^T, then dS^T
//   warps 8-11  dQ warpgroup: drains each query tile's dQ from tensor memory
//               into shared memory and adds it into the fp32 accumulator
//               with bulk reduce-adds, concurrently with the compute warps;
//               at the end of a unit it writes the key tile's dK and dV
//   warp  12    TMA producer      warp 13  MMA issuer      warps 14-15 idle
//   (d = 128: warp 13 issues dP, dK, dQ and warp 14 issues S, dV, with the
//   unit's K tile copied into tensor memory as the A operand of S^T)
// An issuer runs barely ahead of the tensor core, so each of its waits and
// each piece of its bookkeeping leaves the tensor core idle.  At d = 128 the
// products are split over two issuers with disjoint tensor-memory regions,
// so one issues while the other waits, and each waits once per query tile
// (A for dS, B for P), the other conditions being folded into those
// barriers (kFoldWaits, kTwoIssuers).
#include <cuda_fp16.h>

#include <type_traits>

#include "sm100_ptx.cuh"
#include "fa_kernels.h"

namespace fa {

namespace {

constexpr int kBwdThreads = 512;
constexpr int kBDqWarp0 = 8;         // warps 8-11: dQ warpgroup (TMEM lane quadrants 0-3)
constexpr int kBProducerWarp = 12;
constexpr int kBMmaWarp = 13;
// Register split: every SM sub-partition holds one warp of each warpgroup
// (warp w runs on sub-partition w % 4): two compute warps, one dQ warp and
// one of the producer / MMA / idle warpgroup.
constexpr int kBLaunchRegs = 128;
constexpr int kBRegsCompute = 136;
constexpr int kBRegsDq = 120;
constexpr int kBRegsOther = 120;
static_assert(2 * kBRegsCompute + kBRegsDq + kBRegsOther <= 4 * kBLaunchRegs,
              "register split exceeds a sub-partition's pool");

template <int D>
struct BwdLayout {
  static constexpr int BR = (D == 64) ? 128 : 64;  // query rows per tile
  static constexpr int kKV = kBlockN * D * 2;      // K or V tile bytes
  static constexpr int kQT = BR * D * 2;           // Q or dO tile bytes
  static constexpr int kDS = kBlockN * BR * 2;     // dS^T tile bytes
  // fp32 dQ staging.  d = 64: one padded row per query (272-byte pitch, so
  // that the eight rows of a 16-byte store phase start on different banks),
  // each row added to the accumulator by its own thread; d = 128: the
  // [64 queries][128 dims] tile, contiguous, added with one bulk reduce.
  static constexpr int kStgPitch = (D == 64) ? D * 4 + 16 : D * 4;
  static constexpr int kStage = BR * kStgPitch;
  // K/V buffers: two at d = 64, so that the next unit's key/value tiles load
  // while the current unit runs (units of short sequences are a few
  // iterations long); the Q/dO ring is then 2 deep to stay within shared
  // memory.  d = 128 (32 KB tiles): one K/V buffer, a 3-deep ring.
  static constexpr int kKVBufs = (D == 64) ? 2 : 1;
  static constexpr int kKOff = 0;                  // buffer b: K at b * 2 kKV, V after it
  static constexpr int kVOff = kKOff + kKV;
  static constexpr int kStages = (D == 64) ? 2 : 3;  // Q / dO / LSE / D ring depth
  // d = 128 (3-deep ring): the MMA issuer's per-tile waits are folded into
  // the two it must make anyway.  kPFull also means "the next tile's Q/dO
  // have landed" (the compute warpgroups wait for them first) and kDSFull
  // also means "dQ of the previous tile has left tensor memory" (the dQ
  // warpgroup arrives on it).  With the 2-deep ring of d = 64 the next tile
  // is often still loading when P is ready, so there the issuer waits on
  // kQFull and kDQEmpty itself.
  static constexpr bool kFoldWaits = (D == 128);
  // d = 128: two MMA issuers, so that one issues while the other waits.
  // Issuer A (warp 13) owns the dP region and the dK / dQ accumulators
  // (dP, dK, dQ; waits on kDSFull), issuer B (warp 14) the S region and dV
  // (S, dV; waits on kPFull).  Their products touch disjoint tensor-memory
  // columns, so the tensor core may interleave the two streams in any order;
  // within each stream a thread's MMAs run in issue order.  Barriers that
  // both streams release (Q/dO stage, K/V tiles, accumulators, drain) count
  // one commit per issuer.
  static constexpr bool kTwoIssuers = kFoldWaits;
  static constexpr int kIssuers = kTwoIssuers ? 2 : 1;
  static constexpr int kQOff = kKVBufs * 2 * kKV;    // [kStages]
  static constexpr int kDOOff = kQOff + kStages * kQT;
  static constexpr int kDSOff = kDOOff + kStages * kQT;
  // d = 128 (two issuers): two dS^T shared tiles, so that the compute
  // warpgroups write tile i's while dQ(i-1) still reads tile i-1's
  static constexpr int kDSBufs = (D == 128) ? 2 : 1;
  static constexpr int kStgOff = kDSOff + kDSBufs * kDS;
  static constexpr int kVecOff = kStgOff + kStage;  // [kStages] x (nlse2[BR], dvec[BR])
  static constexpr int kVecStage = 2 * BR * 4;
  static constexpr int kBarOff = kVecOff + kStages * kVecStage;
  // barriers
  static constexpr int kKVFull = 0, kKVEmpty = kKVBufs;   // [kKVBufs] each
  static constexpr int kQFull = 2 * kKVBufs;             // [kStages]
  static constexpr int kQEmpty = kQFull + kStages;  // [kStages]
  static constexpr int kSFull = kQEmpty + kStages, kDPFull = kSFull + 1, kPFull = kSFull + 2;
  static constexpr int kDSFull = kSFull + 3, kDSEmpty = kSFull + 4, kDQFull = kSFull + 5;
  static constexpr int kDQEmpty = kSFull + 6, kAccFull = kSFull + 7, kAccEmpty = kSFull + 8, kDrain = kSFull + 9;
  // dQ staging tile: free again (previous reduce has read it) / fully written
  static constexpr int kStgFree = kSFull + 10, kStgDone = kSFull + 11;
  static constexpr int kDSEmpty1 = kSFull + 12;   // dS^T shared tile 1 read (two tiles)
  static constexpr int kNumBars = kDSEmpty1 + 1;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kBytes = kMiscOff + 16;
  static constexpr int kAlloc = kBytes + 1024;
  // tensor-memory columns
  static constexpr uint32_t kColS = 0;
  static constexpr uint32_t kColDP = BR;
  static constexpr uint32_t kColDV = 2 * BR;
  static constexpr uint32_t kColDK = 2 * BR + D;
  static constexpr uint32_t kColDQ = 2 * BR + 2 * D;
  // two issuers (d = 128): the unit's K tile is copied into the last 64
  // columns, so that S^T reads only Q from shared memory
  static constexpr uint32_t kColK = kColDQ + BR;
  static_assert(!kFoldWaits || kColK + D / 2 <= 512, "tensor memory overflow");
  static_assert(kColDQ + (D == 64 ? D : BR) <= 512, "tensor memory overflow");
  // Compute warpgroup w (0, 1) owns query columns [w*HALF, (w+1)*HALF) of
  // each tile and packs its 16-bit P^T / dS^T (two per 32-bit column) at the
  // start of that range, so the two warpgroups never write columns the other
  // still reads.  Column of the 16 queries of MMA K step ks:
  static constexpr int HALF = BR / 2;
  __host__ __device__ static constexpr uint32_t packed_col(int ks) {
    return (uint32_t)((ks / (HALF / 16)) * HALF + (ks % (HALF / 16)) * 8);
  }
  static_assert(kAlloc <= 232448, "shared memory overflow");
};

struct BUnit {
  int kvbh;   // batch * Hkv + key/value head
  int qbh0;   // batch * H + first query head of the group
  int jk;     // key tile
  int i0;     // first query tile (causal: the diagonal one)
  int n_i;    // query tiles per query head
  int n_it;   // iterations: group x n_i (query head major)
  __device__ __forceinline__ int qbh(int it) const { return qbh0 + it / n_i; }
  __device__ __forceinline__ int qtile(int it) const { return i0 + it % n_i; }
};

// Unit = (batch, key/value head, 128-key tile).  Its iterations run over the
// query heads that share the key/value head (grouped-query attention; one
// head when H = Hkv) and, for each, over the query tiles that see the key
// tile, so dK and dV accumulate over the whole group in tensor memory.
template <int D, bool CAUSAL>
__device__ __forceinline__ BUnit decode_bunit(int u, const BwdParams& p) {
  constexpr int BR = BwdLayout<D>::BR;
  BUnit r;
  const int bhkv = p.bh / p.group;  // B * Hkv
  if (CAUSAL) {  // key tile 0 has the most query tiles: longest first
    r.jk = u / bhkv;
    r.kvbh = u % bhkv;
  } else {       // neighbouring CTAs share a head (Q / dO reuse in L2)
    r.jk = u % p.n_kv;
    r.kvbh = u / p.n_kv;
  }
  r.qbh0 = r.kvbh * p.group;  // (b * Hkv + hkv) * group = b * H + hkv * group
  r.i0 = CAUSAL ? (r.jk * kBlockN) / BR : 0;
  r.n_i = (p.N + BR - 1) / BR - r.i0;
  r.n_it = r.n_i * p.group;
  return r;
}

// Whether iteration `it` of the unit is computed: its query block attends the
// unit's key block (always when dense).  The mask bytes of 32 iterations are
// fetched at once (independent loads) into a register window; a role that
// walks its iterations forward loads each window once.
struct IterWin {
  int base = -32;
  uint32_t bits = 0;
};
template <int D, bool SPARSE>
__device__ __forceinline__ bool bactive(IterWin& w, const BwdParams& p, const BUnit& bu, int it) {
  if constexpr (!SPARSE) return true;
  constexpr int BR = BwdLayout<D>::BR;
  if (it < w.base || it >= w.base + 32) {
    w.base = it & ~31;
    w.bits = 0;
#pragma unroll 8
    for (int i = 0; i < 32; ++i) {
      const int t = w.base + i;
      if (t < bu.n_it) {
        const int qblk = (bu.qtile(t) * BR) / kBlockN;
        if (p.bmask[(long long)bu.qbh(t) * p.bmask_stride + (long long)qblk * p.n_kv + bu.jk] != 0) w.bits |= 1u << i;
      }
    }
  }
  return (w.bits >> (it - w.base)) & 1u;
}

// Tile of R rows x D columns stored as D/64 column blocks of R x 128 B (SW128).
// K-major operand view: advance 16 elements (32 B) per K step.
template <int R>
__device__ __forceinline__ uint64_t kmaj(uint32_t tile, int kstep) {
  return make_sdesc_sw128(tile + (uint32_t)(kstep >> 2) * (R * 128) + (uint32_t)(kstep & 3) * 32, 16, 1024);
}
// MN-major operand view of the same storage (MN = the 64-wide column axis,
// K = the row axis): column blocks R*128 bytes apart, 16 rows per K step.
template <int R>
__device__ __forceinline__ uint64_t mnmaj(uint32_t tile, int kstep) {
  return make_sdesc_sw128(tile + (uint32_t)kstep * 2048, R * 128, 1024);
}
// Byte offsets of K step `kstep` in the two views (for sdesc_advance: the MMA
// issuer builds each descriptor once and steps it by these constants).
template <int R>
__host__ __device__ constexpr uint32_t kmaj_off(int kstep) {
  return (uint32_t)(kstep >> 2) * (R * 128) + (uint32_t)(kstep & 3) * 32;
}
__host__ __device__ constexpr uint32_t mnmaj_off(int kstep) { return (uint32_t)kstep * 2048; }

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
               : "memory");
}
__device__ __forceinline__ void bulk_reduce_add_f32(float* dst, uint32_t src, uint32_t bytes) {
  asm volatile("cp.reduce.async.bulk.global.shared::cta.bulk_group.add.f32 [%0], [%1], %2;" ::"l"(
                   reinterpret_cast<uint64_t>(dst)),
               "r"(src), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

template <int D, bool BF16, bool CAUSAL, bool SPARSE>
__global__ void __launch_bounds__(kBwdThreads, 1)
    fa_bwd_main(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                const BwdParams p) {
  using L = BwdLayout<D>;
  constexpr int BR = L::BR;
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
    for (int b = 0; b < L::kKVBufs; ++b) {
      mbar_init(BAR(L::kKVFull + b), 1);
      mbar_init(BAR(L::kKVEmpty + b), L::kIssuers);
    }
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(BAR(L::kQFull + s), 1);
      mbar_init(BAR(L::kQEmpty + s), L::kIssuers);
    }
    mbar_init(BAR(L::kSFull), 1);
    mbar_init(BAR(L::kDPFull), 1);
    mbar_init(BAR(L::kPFull), 256);
    // dS^T of tile i written (256 compute threads) and, folded, dQ of tile
    // i-1 read out of tensor memory (128 dQ-warpgroup threads)
    mbar_init(BAR(L::kDSFull), L::kFoldWaits ? 384 : 256);
    mbar_init(BAR(L::kDQEmpty), 128);
    mbar_init(BAR(L::kDSEmpty), 1);
    mbar_init(BAR(L::kDSEmpty1), 1);
    mbar_init(BAR(L::kDQFull), 1);
    mbar_init(BAR(L::kAccFull), L::kIssuers);
    mbar_init(BAR(L::kAccEmpty), 128);
    mbar_init(BAR(L::kDrain), L::kIssuers);
    mbar_init(BAR(L::kStgFree), 1);
    mbar_init(BAR(L::kStgDone), 128);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kBProducerWarp) {
    tmem_alloc(smem_u32(const_cast<uint32_t*>(tmem_slot)), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtx wc{p.wait_limit_ns, abort_flag, p.status};
  // nothing above touched global memory; D, -LSE*log2e and the zeroed dQ
  // accumulator come from the preparation kernel
  grid_dependency_wait();
  grid_dependents_launch();
  if (warp >= kBProducerWarp) regs_dec<kBRegsOther>();
  else if (warp >= kBDqWarp0) regs_dec<kBRegsDq>();
  else regs_inc<kBRegsCompute>();

  if (warp == kBProducerWarp) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmDO);
      // K, V: read once per unit.  Q, dO: re-read by every unit of the head
      // (the CTAs working on one head run at about the same pace, so the
      // reuse is close in time); normal priority, so that they do not push
      // the fp32 dQ accumulator, reduce-added by the same CTAs, out of L2.
      const uint64_t pol_kv = l2_policy_evict_first();
      const uint64_t pol_q = l2_policy_evict_normal();
      uint32_t unit_iter = 0, q_iter = 0, kv_issued = 0;
      bool ok = true;
      for (int k = 0, u = unit_of(0); u < p.n_units && ok; u = unit_of(++k), ++unit_iter) {
        const BUnit bu = decode_bunit<D, CAUSAL>(u, p);
        const uint32_t kb = unit_iter % L::kKVBufs, kuse = unit_iter / L::kKVBufs;
        if (kuse > 0 && !mbar_wait(BAR(L::kKVEmpty + kb), (kuse - 1) & 1, wc)) { ok = false; break; }
        mbar_arrive_expect_tx(BAR(L::kKVFull + kb), 2 * L::kKV);
        const uint32_t kvb = base + kb * 2 * L::kKV;
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          tma_load_3d(kvb + L::kKOff + c * (kBlockN * 128), &tmK, BAR(L::kKVFull + kb), c * 64, bu.jk * kBlockN, bu.kvbh,
                      pol_kv);
          tma_load_3d(kvb + L::kVOff + c * (kBlockN * 128), &tmV, BAR(L::kKVFull + kb), c * 64, bu.jk * kBlockN, bu.kvbh,
                      pol_kv);
        }
        ++kv_issued;
        IterWin iw;
        for (int it = 0; it < bu.n_it; ++it) {
          if (!bactive<D, SPARSE>(iw, p, bu, it)) continue;
          const int i = bu.qtile(it), qbh = bu.qbh(it);
          const uint32_t st = q_iter % L::kStages, use = q_iter / L::kStages;
          if (use > 0 && !mbar_wait(BAR(L::kQEmpty + st), (use - 1) & 1, wc)) { ok = false; break; }
          const uint32_t fb = BAR(L::kQFull + st);
          mbar_arrive_expect_tx(fb, 2 * L::kQT + L::kVecStage);
#pragma unroll
          for (int c = 0; c < D / 64; ++c) {
            tma_load_3d(base + L::kQOff + st * L::kQT + c * (BR * 128), &tmQ, fb, c * 64, i * BR, qbh, pol_q);
            tma_load_3d(base + L::kDOOff + st * L::kQT + c * (BR * 128), &tmDO, fb, c * 64, i * BR, qbh, pol_q);
          }
          const size_t row0 = (size_t)qbh * p.n_pad + (size_t)i * BR;
          bulk_load(base + L::kVecOff + st * L::kVecStage, p.nlse2 + row0, BR * 4, fb);
          bulk_load(base + L::kVecOff + st * L::kVecStage + BR * 4, p.dvec + row0, BR * 4, fb);
          ++q_iter;
        }
      }
      if (!ok) {
        // Let every copy already issued land before the CTA exits.
        for (uint32_t b = 0; b < (uint32_t)L::kKVBufs; ++b) {
          const uint32_t issued = kv_issued / L::kKVBufs + (b < kv_issued % L::kKVBufs ? 1u : 0u);
          if (issued > 0) mbar_wait_drain(BAR(L::kKVFull + b), (issued - 1) & 1, p.wait_limit_ns);
        }
        for (uint32_t s = 0; s < (uint32_t)L::kStages; ++s) {
          const uint32_t issued = q_iter / L::kStages + (s < q_iter % L::kStages ? 1u : 0u);
          if (issued > 0) mbar_wait_drain(BAR(L::kQFull + s), (issued - 1) & 1, p.wait_limit_ns);
        }
      }
    }
  } else if (warp == kBMmaWarp || (L::kTwoIssuers && warp == kBMmaWarp + 1)) {
    // ---------------------------------------------------------------- MMA
    // role 0: the single issuer (d = 64); 1: issuer A (dP, dK, dQ); 2: issuer
    // B (S, dV)
    const int role = L::kTwoIssuers ? (warp == kBMmaWarp ? 1 : 2) : 0;
    const bool do_a = role != 2, do_b = role != 1;
    if (lane == 0) {
      constexpr uint32_t idesc_s = make_idesc_f16(BF16, kBlockN, BR, false, false);   // S^T, dP^T
      constexpr uint32_t idesc_acc = make_idesc_f16(BF16, kBlockN, D, false, true);   // dV, dK
      // dQ (d=64: M=128 queries, N=64) or dQ^T (d=128: M=128 dims, N=64 queries)
      constexpr uint32_t idesc_dq = make_idesc_f16(BF16, 128, 64, true, true);
      uint32_t unit_iter = 0, p_cnt = 0, ds_cnt = 0, dq_cnt = 0;
      // The issuer runs barely ahead of the tensor core, so its bookkeeping
      // between products is kept short: the Q/dO descriptors of ring stage
      // s are stage 0's advanced by s * kQT bytes, and the stage index and
      // its phase are stepped, not divided out of a tile counter.
      const uint64_t dQ0 = kmaj<BR>(base + L::kQOff, 0), dDO0 = kmaj<BR>(base + L::kDOOff, 0);
      const uint64_t dQmn0 = mnmaj<BR>(base + L::kQOff, 0), dDOmn0 = mnmaj<BR>(base + L::kDOOff, 0);
      uint32_t st = 0, st_ph = 0;  // ring stage of the current tile and the parity of its use
      auto next_stage = [](uint32_t s0, uint32_t ph0, uint32_t& s1, uint32_t& ph1) {
        s1 = s0 + 1 == (uint32_t)L::kStages ? 0u : s0 + 1;
        ph1 = s1 == 0 ? ph0 ^ 1u : ph0;
      };
      bool ok = true;
      for (int k = 0, u = unit_of(0); u < p.n_units && ok; u = unit_of(++k), ++unit_iter) {
        const BUnit bu = decode_bunit<D, CAUSAL>(u, p);
        const uint32_t kb = unit_iter % L::kKVBufs;
        if (!mbar_wait(BAR(L::kKVFull + kb), (unit_iter / L::kKVBufs) & 1, wc)) { ok = false; break; }
        const uint32_t sK = base + kb * 2 * L::kKV + L::kKOff, sV = base + kb * 2 * L::kKV + L::kVOff;
        const uint64_t dK = kmaj<kBlockN>(sK, 0), dV = kmaj<kBlockN>(sV, 0), dKmn = mnmaj<kBlockN>(sK, 0);
        const uint64_t dDSmn0 = mnmaj<kBlockN>(base + L::kDSOff, 0);
        IterWin iw;  // walks forward only: the scan for the next iteration leads
        int a0 = 0;  // first computed iteration (n_it when the key tile is attended by none)
        while (a0 < bu.n_it && !bactive<D, SPARSE>(iw, p, bu, a0)) ++a0;
        // S^T (and, issuer A, dP^T) for the first query tile
        if (a0 < bu.n_it) {
          if (!mbar_wait(BAR(L::kQFull + st), st_ph, wc)) { ok = false; break; }
          tc_fence_after();
          if (do_b) {
            const uint64_t dQ = sdesc_advance(dQ0, st * L::kQT);
            if (role == 2) {
              // K into tensor memory, one K step (128 keys x 16 dims) per copy;
              // the previous unit's S^T products, issued earlier by this
              // thread, have read the region before these copies run
#pragma unroll
              for (int ks = 0; ks < D / 16; ++ks)
                tc_cp_128x256b(tmem + L::kColK + 8u * ks, sdesc_advance(dK, kmaj_off<kBlockN>(ks)));
#pragma unroll
              for (int ks = 0; ks < D / 16; ++ks)
                mma_ts(tmem + L::kColS, tmem + L::kColK + 8u * ks, sdesc_advance(dQ, kmaj_off<BR>(ks)), idesc_s,
                       ks > 0);
            } else {
#pragma unroll
              for (int ks = 0; ks < D / 16; ++ks)
                mma_ss(tmem + L::kColS, sdesc_advance(dK, kmaj_off<kBlockN>(ks)), sdesc_advance(dQ, kmaj_off<BR>(ks)),
                       idesc_s, ks > 0);
            }
            tc_commit(BAR(L::kSFull));
          }
          if (role == 1) {
            const uint64_t dDO = sdesc_advance(dDO0, st * L::kQT);
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks)
              mma_ss(tmem + L::kColDP, sdesc_advance(dV, kmaj_off<kBlockN>(ks)), sdesc_advance(dDO, kmaj_off<BR>(ks)),
                     idesc_s, ks > 0);
            tc_commit(BAR(L::kDPFull));
          }
        }
        for (int it = a0, nxt; it < bu.n_it; it = nxt) {  // active iterations only
          const uint32_t soff = st * L::kQT;
          const uint64_t dDO = sdesc_advance(dDO0, soff), dDOmn = sdesc_advance(dDOmn0, soff),
                         dQmn = sdesc_advance(dQmn0, soff);
          uint32_t st1, st1_ph;  // stage of the next tile
          next_stage(st, st_ph, st1, st1_ph);
          const uint32_t first = (it == a0);
          nxt = it + 1;
          while (nxt < bu.n_it && !bactive<D, SPARSE>(iw, p, bu, nxt)) ++nxt;
          if (role == 0) {
            // dP^T = V_j dO_i^T   (the dP region's previous contents, dS^T
            // of tile i-1, were consumed by dK(i-1), issued earlier)
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks)
              mma_ss(tmem + L::kColDP, sdesc_advance(dV, kmaj_off<kBlockN>(ks)), sdesc_advance(dDO, kmaj_off<BR>(ks)),
                     idesc_s, ks > 0);
            tc_commit(BAR(L::kDPFull));
          }
          if (do_b) {
          // dV += P^T dO_i
          if (!mbar_wait(BAR(L::kPFull), p_cnt & 1, wc)) { ok = false; break; }
          ++p_cnt;
          if (first && unit_iter > 0 && !mbar_wait(BAR(L::kAccEmpty), (unit_iter - 1) & 1, wc)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int ks = 0; ks < BR / 16; ++ks)
            mma_ts(tmem + L::kColDV, tmem + L::kColS + L::packed_col(ks), sdesc_advance(dDOmn, mnmaj_off(ks)), idesc_acc,
                   (!first || ks > 0) ? 1u : 0u);
          // S^T for the next query tile (the S region's P^T was consumed by dV
          // above).  Folded: its Q tile has landed, since the compute
          // warpgroups waited for it before arriving on kPFull.
          if (nxt < bu.n_it) {
            if constexpr (!L::kFoldWaits) {
              if (!mbar_wait(BAR(L::kQFull + st1), st1_ph, wc)) { ok = false; break; }
              tc_fence_after();
            }
            const uint64_t dQ1 = sdesc_advance(dQ0, st1 * L::kQT);
            if (role == 2) {
#pragma unroll
              for (int ks = 0; ks < D / 16; ++ks)
                mma_ts(tmem + L::kColS, tmem + L::kColK + 8u * ks, sdesc_advance(dQ1, kmaj_off<BR>(ks)), idesc_s,
                       ks > 0);
            } else {
#pragma unroll
              for (int ks = 0; ks < D / 16; ++ks)
                mma_ss(tmem + L::kColS, sdesc_advance(dK, kmaj_off<kBlockN>(ks)), sdesc_advance(dQ1, kmaj_off<BR>(ks)),
                       idesc_s, ks > 0);
            }
            tc_commit(BAR(L::kSFull));
          }
          }  // do_b
          if (do_a) {
          if (!mbar_wait(BAR(L::kDSFull), ds_cnt & 1, wc)) { ok = false; break; }
          const uint32_t db = L::kDSBufs == 2 ? (ds_cnt & 1u) : 0u;   // dS^T shared tile of this query tile
          const uint64_t dDSmn = sdesc_advance(dDSmn0, db * L::kDS);
          ++ds_cnt;
          if (role == 1 && first && unit_iter > 0 && !mbar_wait(BAR(L::kAccEmpty), (unit_iter - 1) & 1, wc)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // dK += dS^T Q_i
#pragma unroll
          for (int ks = 0; ks < BR / 16; ++ks)
            mma_ts(tmem + L::kColDK, tmem + L::kColDP + L::packed_col(ks), sdesc_advance(dQmn, mnmaj_off(ks)), idesc_acc,
                   (!first || ks > 0) ? 1u : 0u);
          if (role == 1 && nxt < bu.n_it) {
            // dP^T of the next tile (after dK(i), the last reader of the dP
            // region's dS^T; its dO has landed: the compute warpgroups waited
            // for it before arriving on kPFull, and so before kDSFull)
            const uint64_t dDO1 = sdesc_advance(dDO0, st1 * L::kQT);
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks)
              mma_ss(tmem + L::kColDP, sdesc_advance(dV, kmaj_off<kBlockN>(ks)), sdesc_advance(dDO1, kmaj_off<BR>(ks)),
                     idesc_s, ks > 0);
            tc_commit(BAR(L::kDPFull));
          }
          // dQ_i (d=64) or dQ_i^T (d=128) from dS^T in shared memory, once
          // the dQ warpgroup has read dQ_{i-1} out of tensor memory (folded:
          // before its arrival on kDSFull)
          if constexpr (!L::kFoldWaits) {
            if (dq_cnt > 0 && !mbar_wait(BAR(L::kDQEmpty), (dq_cnt - 1) & 1, wc)) { ok = false; break; }
            tc_fence_after();
          }
#pragma unroll
          for (int ks = 0; ks < kBlockN / 16; ++ks) {
            const uint64_t a = sdesc_advance(D == 64 ? dDSmn : dKmn, mnmaj_off(ks));
            const uint64_t b = sdesc_advance(D == 64 ? dKmn : dDSmn, mnmaj_off(ks));
            mma_ss(tmem + L::kColDQ, a, b, idesc_dq, ks > 0);
          }
          tc_commit(BAR(L::kDQFull));
          ++dq_cnt;
          tc_commit(BAR(db ? L::kDSEmpty1 : L::kDSEmpty));   // dS^T shared tile db no longer read
          }  // do_a
          tc_commit(BAR(L::kQEmpty + st));   // Q_i, dO_i, LSE_i, D_i no longer read (this issuer)
          st = st1;
          st_ph = st1_ph;
        }
        if (!ok) break;
        // A unit with no computed iteration never waited for the previous
        // unit's accumulators to be read; wait here, so that the accumulator
        // barrier is never two phases ahead of the warpgroup that reads it.
        if (a0 >= bu.n_it && unit_iter > 0 && !mbar_wait(BAR(L::kAccEmpty), (unit_iter - 1) & 1, wc)) {
          ok = false;
          break;
        }
        tc_commit(BAR(L::kAccFull));
        tc_commit(BAR(L::kKVEmpty + kb));
      }
      tc_commit(BAR(L::kDrain));
      mbar_wait_drain(BAR(L::kDrain), 0, p.wait_limit_ns);
    }
  } else if (warp >= kBDqWarp0 && warp < kBDqWarp0 + 4) {
    // ------------------------------------------------------ dQ warpgroup
    // Walks the same iterations as the MMA issuer.  For each dQ tile: read
    // it from tensor memory (thread = tensor-memory lane: the query row at
    // d = 64, the head dimension at d = 128), release the tensor-memory tile,
    // write it to the fp32 staging buffer and add it into the accumulator
    // (the softmax scale is applied once, when the accumulator is converted).
    const int t = threadIdx.x - 32 * kBDqWarp0;    // 0..127 = tensor-memory lane
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    uint8_t* stage = gbase + L::kStgOff;
    const uint32_t stage_s = base + L::kStgOff;
    uint32_t dq_cnt = 0, unit_iter = 0;
    bool ok = true;
    // Folded waits: the dQ tensor-memory tile is free for the first dQ
    // product, this warpgroup's share of the first kDSFull phase.  Each later
    // arrival (after dQ_i is read out) belongs to the phase of tile i+1,
    // which cannot begin before the issuer has consumed tile i's phase.
    if constexpr (L::kFoldWaits) mbar_arrive(BAR(L::kDSFull));
    for (int k = 0, u = unit_of(0); u < p.n_units && ok; u = unit_of(++k), ++unit_iter) {
      const BUnit bu = decode_bunit<D, CAUSAL>(u, p);
      IterWin iw;
      int n_done = 0;  // iterations computed in this unit
      for (int it = 0; it < bu.n_it; ++it) {
        if (!bactive<D, SPARSE>(iw, p, bu, it)) continue;
        ++n_done;
        const uint32_t phase = dq_cnt & 1;
        ok = warp_all(mbar_wait(BAR(L::kDQFull), phase, wc));
        if (!ok) break;
        ++dq_cnt;
        tc_fence_after();
        uint32_t v[64];
        tmem_ld32(tmem + lane_off + L::kColDQ, v);
        tmem_ld32(tmem + lane_off + L::kColDQ + 32u, v + 32);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(BAR(L::kFoldWaits ? L::kDSFull : L::kDQEmpty));
        float* acc_tile = p.dq_acc + ((size_t)bu.qbh(it) * p.n_pad + (size_t)bu.qtile(it) * BR) * D;
        if constexpr (D == 64) {
          // row t of the [128 queries][64 dims] tile: this thread's own
          // staging row and its own bulk reduce (no cross-thread handshake);
          // its previous reduce must have finished reading the row
          if (dq_cnt > 1) bulk_wait_read0();
          uint8_t* row = stage + t * L::kStgPitch;
#pragma unroll
          for (int c = 0; c < 16; ++c)
            *reinterpret_cast<float4*>(row + 16 * c) =
                make_float4(__uint_as_float(v[4 * c]), __uint_as_float(v[4 * c + 1]), __uint_as_float(v[4 * c + 2]),
                            __uint_as_float(v[4 * c + 3]));
          fence_async_smem();
          bulk_reduce_add_f32(acc_tile + (size_t)t * D, stage_s + t * L::kStgPitch, D * 4);
          bulk_commit();
        } else {
          // column t of the [64 queries][128 dims] tile; one thread adds the
          // whole tile once all 128 have written it.  The warpgroup meets on
          // mbarriers with bounded waits, so a warp that timed out cannot
          // leave the others waiting.
          if (t == 0) {
            bulk_wait_read0();  // the previous reduce has finished reading the tile
            mbar_arrive(BAR(L::kStgFree));
          }
          ok = warp_all(mbar_wait(BAR(L::kStgFree), phase, wc));
          if (!ok) break;
          float* st = reinterpret_cast<float*>(stage);
#pragma unroll
          for (int q = 0; q < 64; ++q) st[q * 128 + t] = __uint_as_float(v[q]);
          fence_async_smem();
          mbar_arrive(BAR(L::kStgDone));
          bool good = true;
          if (t == 0) {
            good = mbar_wait(BAR(L::kStgDone), phase, wc);
            if (good) {
              bulk_reduce_add_f32(acc_tile, stage_s, L::kStage);
              bulk_commit();
            }
          }
          ok = warp_all(good);
          if (!ok) break;
        }
      }
      if (!ok) break;
      // dK, dV of this key tile (lane t = key): read from tensor memory once
      // the unit's last products are done, then released to the next unit's
      // first dV / dK products.  Done here rather than in the compute
      // warpgroups, which go straight on to the next unit's first P.
      ok = warp_all(mbar_wait(BAR(L::kAccFull), unit_iter & 1, wc));
      if (!ok) break;
      tc_fence_after();
      const int key = bu.jk * kBlockN + t;
      const bool in_range = key < p.N;
      const size_t rowoff = ((size_t)bu.kvbh * p.N + (size_t)(in_range ? key : 0)) * D * 2;
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        const uint32_t col = which ? L::kColDK : L::kColDV;
        const float mul = which ? p.scale : 1.f;
        uint8_t* dst = reinterpret_cast<uint8_t*>(which ? p.dk : p.dv) + rowoff;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t r[32];
          if (n_done > 0) {
            tmem_ld32(tmem + lane_off + col + 32u * c, r);
            tmem_wait_ld();
          } else {  // no query attends this key tile: zero gradient
#pragma unroll
            for (int e = 0; e < 32; ++e) r[e] = 0u;
          }
          if (which == 1 && c == D / 32 - 1) {  // every accumulator column has been read
            tc_fence_before();
            mbar_arrive(BAR(L::kAccEmpty));
          }
          uint32_t wv[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            wv[e] = pack2<BF16>(__uint_as_float(r[2 * e]) * mul, __uint_as_float(r[2 * e + 1]) * mul);
          if (in_range) {
            uint4* o = reinterpret_cast<uint4*>(dst + c * 64);
#pragma unroll
            for (int e = 0; e < 4; ++e) o[e] = make_uint4(wv[4 * e], wv[4 * e + 1], wv[4 * e + 2], wv[4 * e + 3]);
          }
        }
      }
    }
    bulk_wait0();  // every reduce this thread issued has landed before the CTA exits
  } else if (warp < 8) {
    // ------------------------------------------------- compute warpgroups 0, 1
    // Both warpgroups run the same loop on their own half of each query tile
    // (queries [w*HALF, (w+1)*HALF)), thread = key = tensor-memory lane:
    //   P^T half, arrive P; dS^T half, arrive dS.  At the end of a unit each
    //   warpgroup writes half of the dims of dK and dV.
    const int w = warp >> 2;                       // 0 or 1
    const int key_in = threadIdx.x & 127;          // tensor-memory lane
    const int tid256 = threadIdx.x;                // 0..255 over both warpgroups
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_off + L::kColS;
    const uint32_t tDP = tmem + lane_off + L::kColDP;
    const float sl2 = p.scale_log2;
    constexpr int HALF = L::HALF;
    constexpr int NC = HALF / 32;                  // 32-column chunks per warpgroup
    uint32_t q_iter = 0, s_cnt = 0, dp_cnt = 0, ds_cnt = 0, unit_iter = 0;
    bool ok = true;

    for (int k = 0, u = unit_of(0); u < p.n_units && ok; u = unit_of(++k), ++unit_iter) {
      const BUnit bu = decode_bunit<D, CAUSAL>(u, p);
      const int key = bu.jk * kBlockN + key_in;
      const bool key_ok = key < p.N;
      IterWin iw;
      bool q_seen = false;  // this tile's Q/dO stage was already waited for
      for (int it = 0; it < bu.n_it; ++it) {
        if (!bactive<D, SPARSE>(iw, p, bu, it)) continue;
        const int i = bu.qtile(it);
        const uint32_t st = q_iter % L::kStages;
        if (!q_seen) {
          ok = warp_all(mbar_wait(BAR(L::kQFull + st), (q_iter / L::kStages) & 1, wc));
          if (!ok) break;
        }
        // this half's -LSE*log2e and D, read four at a time (16-byte aligned)
        const float4* nlse2 = reinterpret_cast<const float4*>(gbase + L::kVecOff + st * L::kVecStage) + HALF * w / 4;
        const float4* dvec = nlse2 + BR / 4;
        const uint64_t sl2x2 = f2_pack(sl2, sl2);
        ok = warp_all(mbar_wait(BAR(L::kSFull), s_cnt & 1, wc));
        if (!ok) break;
        ++s_cnt;
        tc_fence_after();
        const int q0 = i * BR + HALF * w;  // first query of this warpgroup's half
        // P^T = exp2(S^T * scale*log2e - LSE*log2e), masked; kept packed.
        // Only the key tile that holds the last keys (ragged) and, causal,
        // tiles with a key after this half's first query need the mask: the
        // test is uniform over the warpgroup, and the other tiles take the
        // loop without the per-element compare and select.
        const bool need_mask = (bu.jk + 1) * kBlockN > p.N || (CAUSAL && (bu.jk + 1) * kBlockN - 1 > q0);
        uint32_t pk[HALF / 2];
        auto p_half = [&](auto masked) {
#pragma unroll
          for (int c = 0; c < NC; ++c) {
            uint32_t r[32];
            tmem_ld32(tS + HALF * w + 32u * c, r);
            tmem_wait_ld();
            float4 lq;
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const int qa = 32 * c + 2 * e;
              if ((e & 1) == 0) lq = nlse2[qa >> 2];
              // both exponents of the pair in one two-wide fma
              float x0, x1;
              f2_unpack(f2_fma(f2_pack(__uint_as_float(r[2 * e]), __uint_as_float(r[2 * e + 1])), sl2x2,
                               (e & 1) ? f2_pack(lq.z, lq.w) : f2_pack(lq.x, lq.y)),
                        x0, x1);
              float p0 = ex2_approx(x0);
              float p1 = ex2_approx(x1);
              if constexpr (decltype(masked)::value) {
                if (!key_ok || (CAUSAL && key > q0 + qa)) p0 = 0.f;
                if (!key_ok || (CAUSAL && key > q0 + qa + 1)) p1 = 0.f;
              }
              pk[16 * c + e] = pack2<BF16>(p0, p1);
            }
          }
        };
        if (need_mask)
          p_half(std::true_type{});
        else
          p_half(std::false_type{});
        // packed P^T of this half -> columns [HALF*w, HALF*w + HALF/2) of the
        // S^T region, all of which this warpgroup has already read
#pragma unroll
        for (int c = 0; c < NC; ++c) tmem_st16(tS + HALF * w + 16u * c, pk + 16 * c);
        tmem_wait_st();
        tc_fence_before();
        // Folded waits: the issuer computes the next tile's S^T right after
        // dV; wait here for that tile's Q, so the issuer needs no wait of its
        // own.  (The scan moves the mask window forward; the loop's own test
        // of the next iterations then refetches it.)
        if constexpr (L::kFoldWaits) {
          int nxt = it + 1;
          while (nxt < bu.n_it && !bactive<D, SPARSE>(iw, p, bu, nxt)) ++nxt;
          q_seen = nxt < bu.n_it;
        }
        if (q_seen) {
          const uint32_t q1 = q_iter + 1;
          ok = warp_all(mbar_wait(BAR(L::kQFull + q1 % L::kStages), (q1 / L::kStages) & 1, wc));
          if (!ok) break;
        }
        const bool withhold = (p.debug_flags & 2) && unit_iter == 0 && q_iter == 0 && tid256 == 0;
        if (!withhold) mbar_arrive(BAR(L::kPFull));
        // dS^T = P^T o (dP^T - D)
        ok = warp_all(mbar_wait(BAR(L::kDPFull), dp_cnt & 1, wc));
        if (!ok) break;
        ++dp_cnt;
        tc_fence_after();
        // the dS^T shared tile this query tile writes has been read by its
        // previous dQ product (two tiles: the one two query tiles back)
        const uint32_t db = L::kDSBufs == 2 ? (ds_cnt & 1u) : 0u;
        if constexpr (L::kDSBufs == 2)
          ok = warp_all(ds_cnt < 2 || mbar_wait(BAR(db ? L::kDSEmpty1 : L::kDSEmpty), ((ds_cnt >> 1) - 1) & 1, wc));
        else
          ok = warp_all(ds_cnt == 0 || mbar_wait(BAR(L::kDSEmpty), (ds_cnt - 1) & 1, wc));
        if (!ok) break;
        ++ds_cnt;
        // dS^T chunk by chunk into tensor memory (for the dK MMA) and into the
        // SW128 shared tile [key][query] (for the dQ MMA).  In the shared tile
        // column block cb holds queries 64cb..64cb+63; 16-byte chunk ch of row
        // key_in lives at position ch ^ (key_in & 7).  Packed dS^T chunk c goes
        // to columns [HALF*w + 16c, +16): dP^T chunk c/2 of this half, read.
        uint8_t* ds_tile = gbase + L::kDSOff + db * L::kDS;
#pragma unroll
        for (int c = 0; c < NC; ++c) {
          uint32_t r[32];
          tmem_ld32(tDP + HALF * w + 32u * c, r);
          tmem_wait_ld();
          uint32_t dsk[16];
          float4 dq4;
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int qa = 32 * c + 2 * e;
            if ((e & 1) == 0) dq4 = dvec[qa >> 2];
            const uint32_t pp = pk[16 * c + e];
            float p0, p1;
            if constexpr (BF16) {
              p0 = __uint_as_float(pp << 16);
              p1 = __uint_as_float(pp & 0xFFFF0000u);
            } else {
              const __half2 h = *reinterpret_cast<const __half2*>(&pp);
              p0 = __low2float(h);
              p1 = __high2float(h);
            }
            // dS = P (dP - D) for the pair in two two-wide instructions
            float ds0, ds1;
            f2_unpack(f2_mul(f2_pack(p0, p1),
                             f2_sub(f2_pack(__uint_as_float(r[2 * e]), __uint_as_float(r[2 * e + 1])),
                                    (e & 1) ? f2_pack(dq4.z, dq4.w) : f2_pack(dq4.x, dq4.y))),
                      ds0, ds1);
            dsk[e] = pack2<BF16>(ds0, ds1);
          }
          tmem_st16(tDP + HALF * w + 16u * c, dsk);
          const int qcol = HALF * w + 32 * c;  // first query of this chunk within the tile
          const int cb = qcol >> 6;
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            const int ch = ((qcol & 63) >> 3) + h;
            uint4 val = make_uint4(dsk[4 * h], dsk[4 * h + 1], dsk[4 * h + 2], dsk[4 * h + 3]);
            *reinterpret_cast<uint4*>(ds_tile + cb * (kBlockN * 128) + key_in * 128 + ((ch ^ (key_in & 7)) * 16)) = val;
          }
        }
        tmem_wait_st();
        fence_async_smem();
        tc_fence_before();
        mbar_arrive(BAR(L::kDSFull));
        ++q_iter;
      }
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == kBProducerWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// D_i = sum_c dO_ic O_ic and LSE_i * log2(e) per row (+inf on the padding
// rows N..n_pad-1 and on rows with LSE = -inf), and the rows of dQacc zeroed.
// D / 8 lanes per row, 8 elements (16 bytes of 16-bit data) per lane, so a
// warp covers 32 / (D / 8) rows per pass with 16-byte accesses; warps stride
// over the row groups.  O is read as 16-bit, or as fp32 for the O32 codes.
template <int D, bool BF16, bool O32>
__global__ void __launch_bounds__(256) fa_bwd_prep(const BwdParams p) {
  grid_dependency_wait();  // O, dO and LSE from the kernels before; the workspace free again
  grid_dependents_launch();
  constexpr int L = D / 8;            // lanes per row
  constexpr int RPW = 32 / L;         // rows per warp pass
  const int lane = threadIdx.x & 31;
  const int sub = lane % L, rsub = lane / L;
  const long long groups = ((long long)p.bh * p.n_pad + RPW - 1) / RPW;
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long g = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); g < groups; g += warps) {
    const long long prow = g * RPW + rsub;           // bh * n_pad + row
    const bool valid = prow < (long long)p.bh * p.n_pad;
    const int bh = valid ? (int)(prow / p.n_pad) : 0;
    const int row = valid ? (int)(prow % p.n_pad) : p.n_pad;
    float acc = 0.f;
    if (valid && row < p.N) {
      const size_t off = ((size_t)bh * p.N + row) * D + (size_t)sub * 8;
      const uint4 dw = *reinterpret_cast<const uint4*>(reinterpret_cast<const uint8_t*>(p.dout) + off * 2);
      float dv[8], ov[8];
      const uint32_t dws[4] = {dw.x, dw.y, dw.z, dw.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if constexpr (BF16) {
          dv[2 * e] = __uint_as_float(dws[e] << 16);
          dv[2 * e + 1] = __uint_as_float(dws[e] & 0xFFFF0000u);
        } else {
          dv[2 * e] = __half2float(__ushort_as_half((unsigned short)(dws[e] & 0xFFFFu)));
          dv[2 * e + 1] = __half2float(__ushort_as_half((unsigned short)(dws[e] >> 16)));
        }
      }
      if constexpr (O32) {
        const float4* o4 = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(p.o) + off);
        const float4 a = o4[0], b = o4[1];
        ov[0] = a.x; ov[1] = a.y; ov[2] = a.z; ov[3] = a.w;
        ov[4] = b.x; ov[5] = b.y; ov[6] = b.z; ov[7] = b.w;
      } else {
        const uint4 ow = *reinterpret_cast<const uint4*>(reinterpret_cast<const uint8_t*>(p.o) + off * 2);
        const uint32_t ows[4] = {ow.x, ow.y, ow.z, ow.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          if constexpr (BF16) {
            ov[2 * e] = __uint_as_float(ows[e] << 16);
            ov[2 * e + 1] = __uint_as_float(ows[e] & 0xFFFF0000u);
          } else {
            ov[2 * e] = __half2float(__ushort_as_half((unsigned short)(ows[e] & 0xFFFFu)));
            ov[2 * e + 1] = __half2float(__ushort_as_half((unsigned short)(ows[e] >> 16)));
          }
        }
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) acc = fmaf(ov[e], dv[e], acc);
    }
#pragma unroll
    for (int s = L / 2; s > 0; s >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, s);
    if (valid) {
      if (sub == 0) {
        p.dvec[prow] = acc;
        // padding rows and rows with no kept key (LSE = -inf, block-sparse)
        // get -inf, so that any P recomputed for them is 0
        const float l = row < p.N ? p.lse[(size_t)bh * p.N + row] : -INFINITY;
        p.nlse2[prow] = l > -INFINITY ? -(l * 1.4426950408889634f) : -INFINITY;
      }
      float4* acc_row = reinterpret_cast<float4*>(p.dq_acc + prow * D) + 2 * sub;
      acc_row[0] = make_float4(0.f, 0.f, 0.f, 0.f);
      acc_row[1] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
}

// dQ = dtype(dQacc) for the real rows.  One thread per 8 elements.
template <int D, bool BF16>
__global__ void __launch_bounds__(256) fa_bwd_dq(const BwdParams p) {
  grid_dependency_wait();  // every reduce into the accumulator has landed
  grid_dependents_launch();
  const size_t idx = (size_t)blockIdx.x * blockDim.x + threadIdx.x;  // 8-element group
  const size_t groups = (size_t)p.bh * p.N * (D / 8);
  if (idx >= groups) return;
  const size_t row = idx / (D / 8);  // bh * N + n
  const int g = (int)(idx % (D / 8));
  const size_t bh = row / p.N, n = row % p.N;
  const float4* src = reinterpret_cast<const float4*>(p.dq_acc + (bh * p.n_pad + n) * D + g * 8);
  const float4 a = src[0], b = src[1];
  const float c = p.scale;  // the accumulator holds dS K without the softmax scale
  uint4 w = make_uint4(pack2<BF16>(a.x * c, a.y * c), pack2<BF16>(a.z * c, a.w * c), pack2<BF16>(b.x * c, b.y * c),
                       pack2<BF16>(b.z * c, b.w * c));
  reinterpret_cast<uint4*>(p.dq)[idx] = w;
}

template <int D, bool BF16, bool CAUSAL>
cudaError_t launch_bwd_t(bool o32, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                         const CUtensorMap& tdo, const BwdParams& p, int grid, cudaStream_t st,
                         cudaEvent_t const* ev_main) {
  {
    // row groups of 32 / (D / 8) rows per warp; a grid of up to 16 blocks of
    // 8 warps per SM strides over them
    const long long groups = ((long long)p.bh * p.n_pad + 32 / (D / 8) - 1) / (32 / (D / 8));
    const long long want = (groups + 7) / 8;
    const int blocks = (int)(want < 148LL * 16 ? want : 148LL * 16);
    cudaError_t e = o32 ? launch_chained(fa_bwd_prep<D, BF16, true>, dim3(blocks), dim3(256), 0, st, p)
                        : launch_chained(fa_bwd_prep<D, BF16, false>, dim3(blocks), dim3(256), 0, st, p);
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  {
    auto kern = p.bmask ? fa_bwd_main<D, BF16, CAUSAL, true> : fa_bwd_main<D, BF16, CAUSAL, false>;
    constexpr int smem = BwdLayout<D>::kAlloc;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    if (ev_main && ev_main[0] && (e = cudaEventRecord(ev_main[0], st)) != cudaSuccess) return e;
    e = launch_chained(kern, dim3(grid), dim3(kBwdThreads), smem, st, tq, tk, tv, tdo, p);
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (ev_main && ev_main[1] && (e = cudaEventRecord(ev_main[1], st)) != cudaSuccess) return e;
  }
  {
    const long long groups = (long long)p.bh * p.N * (D / 8);
    const int blocks = (int)((groups + 255) / 256);
    cudaError_t e = launch_chained(fa_bwd_dq<D, BF16>, dim3(blocks), dim3(256), 0, st, p);
    return e != cudaSuccess ? e : cudaGetLastError();
  }
}

}  // namespace

int bwd_threads() { return kBwdThreads; }

cudaError_t launch_bwd(int d, bool bf16, bool o32, bool causal, const CUtensorMap& tq, const CUtensorMap& tk,
                       const CUtensorMap& tv, const CUtensorMap& tdo, const BwdParams& p, int grid,
                       cudaStream_t st, cudaEvent_t const* ev_main) {
#define FA_BWD_CASE(DD, BB, CC) \
  if (d == DD && bf16 == BB && causal == CC) return launch_bwd_t<DD, BB, CC>(o32, tq, tk, tv, tdo, p, grid, st, ev_main);
  FA_BWD_CASE(64, true, false)
  FA_BWD_CASE(64, true, true)
  FA_BWD_CASE(64, false, false)
  FA_BWD_CASE(64, false, true)
  FA_BWD_CASE(128, true, false)
  FA_BWD_CASE(128, true, true)
  FA_BWD_CASE(128, false, false)
  FA_BWD_CASE(128, false, true)
#undef FA_BWD_CASE
  return cudaErrorInvalidValue;
}

}  // namespace fa
