// attn_pingpong.cuh -- two-tile ("ping-pong") attention forward for sm_100a,
// 16-bit inputs (bf16 or fp16; P is rounded to the input type).
//
// Same operation as attn_kernel.cuh ("Core 注意力" section "选择最窄的入口";
// "MLA Prefill" parameter table).  A CTA owns a 256-row work unit: two
// 128-row query tiles A and B of one (sequence, head) that share every K and
// V tile.  Each tile has its own TMEM score buffer, its own TMEM output
// accumulator and its own softmax warpgroup; the MMA warp issues
//     PV_A(j-1), S_A(j), PV_B(j-1), S_B(j)
// so the tensor core computes one tile's products while the other tile's
// softmax runs.  S_A(j) overwrites the columns PV_A(j-1) reads P from; it is
// issued after PV_A(j-1) by the same lane, and tcgen05 MMAs from one thread
// execute in issue order.  The same ordering also means that when a softmax
// warpgroup sees S_s(j) complete, PV_s(j-1) has completed, so it can rescale
// O_s in TMEM without a further wait.
//
// Warps: 0-3 softmax of tile A (one thread per row), 4-7 softmax of tile B,
// 8 TMA producer, 9 MMA issuer, 10-11 idle (they only complete warpgroup 2 so
// that its register limit can be lowered in favour of the softmax groups).
// The producer and MMA warps run their loops with all 32 lanes (warp-uniform
// control flow) and one elected lane issues the TMA copies, MMAs and commits;
// running the loops in a single-lane branch instead took ~450 rather than
// ~290 cycles to issue one tile's PV (clock64 trace) and 4% longer overall.
// TMEM: S_A [0,128), S_B [128,256), O_A [256,384), O_B [384,512).  Shared
// memory: Q_A, Q_B, then K and V rings (separate depths, so the 192-wide MLA
// tiles still fit).
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

#include "attn_common.cuh"

namespace wf {

constexpr int kPPThreads = 384;            // 3 warpgroups
constexpr uint32_t kPPSoftmaxRegs = 192;    // warpgroups 0 and 1
constexpr uint32_t kPPOtherRegs = 120;       // warpgroup 2: producer, MMA, 2 idle warps
// launch: 384 threads x 168 registers = 64512 >= 2*128*200 + 128*96 = 63488
static_assert(2 * 128 * kPPSoftmaxRegs + 128 * kPPOtherRegs <= kPPThreads * 168, "register split");

// kKind (KernelKind): kKindFuse is the instance that also writes a
// BlockKVCache chunk (key rows [fuse_lo, fuse_hi) read from the chunk and
// stored into the cache), kKindMask the one that reads explicit masks; the
// plain instance (no mask or causal) carries neither's code.
template <typename T, int DQK, int DROPE, int DV, int kKind = kKindPlain>
struct PPCfg {
  static constexpr bool kFuse = kKind == kKindFuse;
  static constexpr bool kMask = kKind == kKindMask;
  static constexpr int kAtomE = 64;                       // bf16 elements per 128-byte row
  static constexpr int kKStep = 16;
  static constexpr int kQAtoms = (DQK + kAtomE - 1) / kAtomE;
  static constexpr int kRAtoms = DROPE / kAtomE;
  static constexpr int kQKAtoms = kQAtoms + kRAtoms;
  static constexpr int kVAtoms = (DV + kAtomE - 1) / kAtomE;
  static constexpr int kAtomBytes = 128 * 128;
  static constexpr int kQTileBytes = kQKAtoms * kAtomBytes;
  static constexpr int kQBytes = 2 * kQTileBytes;
  static constexpr int kKBytes = kQKAtoms * kAtomBytes;
  static constexpr int kVBytes = kVAtoms * kAtomBytes;
  static constexpr int kBudget = 227 * 1024 - 2048;
  static constexpr int kEqFit = (kBudget - kQBytes) / (kKBytes + kVBytes);
  static constexpr bool kTwoOne = kEqFit < 2 && (kBudget - kQBytes - 2 * kKBytes - kVBytes) >= 0;
  static constexpr int kKStages = kEqFit >= 3 ? 3 : (kEqFit == 2 ? 2 : (kTwoOne ? 2 : 1));
  static constexpr int kVStages = kEqFit >= 3 ? 3 : (kEqFit == 2 ? 2 : 1);
  static constexpr int kKOff = kQBytes;
  static constexpr int kVOff = kKOff + kKStages * kKBytes;
  // Output staging (p.tma_out): a 4 KB area per softmax warp, its 32 rows x
  // 64 columns of O in bf16 / f16 (128-byte swizzle), stored to global
  // memory by the tensor-memory accelerator one half row at a time; head
  // size 128 only, where it fits beside the rings.
  static constexpr int kStageOff = kVOff + kVStages * kVBytes;
  static constexpr bool kTmaEpi =
      DV == 128 && kStageOff + 8 * 4096 + 1024 + 1024 <= 227 * 1024;
  static constexpr int kCtrlOff = kStageOff + (kTmaEpi ? 8 * 4096 : 0);
  static constexpr int kSmemUsed = kCtrlOff + 1024 + 1024;
  static constexpr int kSmemBytes = kSmemUsed > 120 * 1024 ? kSmemUsed : 120 * 1024;
  static constexpr int kSKStepsQK = DQK / kKStep;
  static constexpr int kSKStepsR = DROPE / kKStep;
  static constexpr int kPVKSteps = kBlockN / kKStep;
  static constexpr int kNPV = kVAtoms * kAtomE;
  static constexpr uint32_t kIdescS = instr_desc(Elem16<T>::kFmt, kBlockM, kBlockN, 0);
  static constexpr uint32_t kIdescPV = instr_desc(Elem16<T>::kFmt, kBlockM, kNPV, 1);
  static constexpr uint32_t kTmemCols = 512;
  // FMA-pipe exp2 share (of 16 columns).  Measured on B200 with waits that
  // suspend instead of spinning, a share of 4/16 cost ~4% at head size 128
  // and more with the 192-wide MLA product, so the MUFU unit does all of them.
  static constexpr int kEmuPer16 = 0;
  // Keys of P handed to the PV product ahead of the rest: the softmax warps
  // store p_0 .. p_{kPSplit-1} and signal p_part before exponentiating the
  // remaining columns, so the MMA warp issues those k-steps of PV while they
  // are computed and only the rest of PV and the next S product stay on the
  // path from the last P value to the next scores.  Measured on B200 (short
  // runs): 80 of 128 keys gave +2.4% on the causal GQA prefill (B 4, 32/8
  // heads, L 4096, D 128), +3.7% on the 64/8-head one at L 16 384 and +0.6% on
  // the rolling cache loop (64, 96 and 112 keys were within 0.5% of 80); with
  // a rope part (MLA) every split cost ~1%, so that instance hands P over whole.
  static constexpr int kPSplit = kRAtoms > 0 ? 0 : 80;
  static_assert(kKStages >= 1 && kVStages >= 1 && kSmemUsed <= 227 * 1024, "smem");
  static_assert(DQK % kKStep == 0 && DV % 32 == 0 && kNPV <= 128, "head dims");
  static_assert(kPSplit % kKStep == 0 && kPSplit >= 0 && kPSplit < kBlockN, "P split");
};

struct PPCtrl {
  uint64_t q_full, q_empty, drain;
  uint64_t s_full[2], p_part[2], p_full[2], o_full[2], o_empty[2];
  uint64_t k_full[3], k_empty[3], v_full[3], v_empty[3];
  uint64_t sched_full[2], sched_empty[2];
  volatile int32_t sched_item[2];
  uint32_t tmem_base;
  volatile int32_t abort;
  TileInfo sched_ti[2][2];        // both sub-tiles of the item in each ring slot
};
static_assert(sizeof(PPCtrl) <= 1024, "control block");

// Work items are handed out at run time: the producer thread takes the next
// item index from a global counter (atomicAdd) and publishes it, with the
// decoded tile coordinates of both sub-tiles, in a two-slot ring; the MMA
// thread and the 8 softmax warps read it from there.  Decoding an item takes
// integer divisions (and, for packed sequences, a search over the work prefix
// sums); done once by the producer, which runs ahead, it stays off the path
// from one item's last PV to the next item's first S.  Items
// are thus processed in their enumeration order (locality first, longest
// unit first) by whichever CTA is free, which keeps the K/V tensors in use at
// one time few and balances the load.  The last CTA to exit resets the
// counters for the next launch on the stream.
constexpr uint32_t kSchedConsumers = 1 + 8;     // MMA warp + one lane per softmax warp

// Bounded wait taken by a whole warp: fails in every lane if it failed in any,
// so the lanes of the producer and MMA warps never diverge.
__device__ __forceinline__ bool bwait_w(uint64_t *bar, uint32_t parity, volatile int32_t *abort,
                                        const AttnParams &p) {
  return __all_sync(0xffffffffu, bwait(bar, parity, abort, p));
}

// Consumer side: the next item (or a value >= the item count at the end) and
// the tile coordinates of sub-tile `sub` (both sub-tiles when sub < 0: ti[0],
// ti[1]; meaningless past the last item).
__device__ __forceinline__ bool pp_next_item(const AttnParams &p, PPCtrl *ctl, uint32_t &it,
                                             int32_t &t, TileInfo *ti, int sub, bool arrive) {
  const uint32_t k = it & 1;
  if (!bwait_w(&ctl->sched_full[k], (it >> 1) & 1, &ctl->abort, p)) return false;
  t = ctl->sched_item[k];
  if (sub < 0) {
    ti[0] = ctl->sched_ti[k][0];
    ti[1] = ctl->sched_ti[k][1];
  } else {
    ti[0] = ctl->sched_ti[k][sub];
  }
  if (arrive) mbar_arrive(&ctl->sched_empty[k]);
  ++it;
  return true;
}

// Dense launches with p.unit_major = W > 0: claims go through the (batch, kv
// head) blocks in order, except the last W blocks, whose items are claimed in
// unit-rank order (the longest unit of each of the W blocks, then the next,
// ...), so that the launch ends on short units.  Mapped here to the index of
// the item in the block-major enumeration that tile_info decodes: within the
// last W blocks claim k = ((j * W + b) * G + head in group) * n_split +
// split; item = ((blk * units + j) * G + head) * n_split + split, blk =
// blocks - W + b.
__device__ __forceinline__ int32_t unit_major_item(const AttnParams &p, int32_t k) {
  const int32_t S = p.n_split > 1 ? p.n_split : 1;
  const int32_t G = p.group, blocks = p.batch * p.hkv, W = p.unit_major;
  const int32_t k0 = (blocks - W) * p.units_per_bh * G * S;
  if (k < k0) return k;
  const int32_t u = (k - k0) / S, sp = (k - k0) - u * S;
  const int32_t q = u / G, hh = u - q * G;
  const int32_t j = q / W, blk = blocks - W + (q - j * W);
  return ((blk * p.units_per_bh + j) * G + hh) * S + sp;
}

// ------------------------------------------------------------------ producer
// Runs on all lanes of warp 8; `leader` (one lane) issues the copies.
template <typename Cfg>
__device__ void pp_producer(const AttnParams &p, uint8_t *smem, PPCtrl *ctl, ProducerLog &log,
                            bool leader) {
  if (leader) {
    tma_prefetch_map(&p.tm_q);
    tma_prefetch_map(&p.tm_k);
    tma_prefetch_map(&p.tm_v);
    if (Cfg::kRAtoms) {
      tma_prefetch_map(&p.tm_qr);
      tma_prefetch_map(&p.tm_kr);
    }
    if (Cfg::kFuse) {
      tma_prefetch_map(&p.tm_kc);
      tma_prefetch_map(&p.tm_vc);
    }
  }
  const int leader_lane = __ffs(__ballot_sync(0xffffffffu, leader)) - 1;
  const int32_t n_units = num_units(p);
  uint32_t g = 0, u = 0;
  log.q_last = -1;
  for (int i = 0; i < 3; ++i) log.k_last[i] = log.v_last[i] = -1;
  bool ok = true;
  bool starve = (p.debug_flags & kDebugStarveFirstK) != 0;

  auto load_k = [&](const TileInfo &ti, int32_t j) -> bool {
    const uint32_t gg = g + j, st = gg % Cfg::kKStages, n = gg / Cfg::kKStages;
    if (!bwait_w(&ctl->k_empty[st], (n + 1) & 1, &ctl->abort, p)) return false;
    if (starve) {                     // debug: never load this K tile
      starve = false;
      return true;
    }
    const int32_t krow = ti.krow + j * kBlockN;
    // rows of the new chunk (fused cache write) come from the chunk itself
    const bool fz = Cfg::kFuse && krow >= p.fuse_lo && krow < p.fuse_hi;
    const CUtensorMap *mk = fz ? &p.tm_kc : &p.tm_k;
    const int32_t ry = fz ? krow - p.fuse_lo : krow;
    uint8_t *dst = smem + Cfg::kKOff + st * Cfg::kKBytes;
    if (leader) {
      mbar_arrive_expect_tx(&ctl->k_full[st], Cfg::kKBytes);
#pragma unroll
      for (int a = 0; a < Cfg::kQAtoms; ++a)
        tma_load_4d(dst + a * Cfg::kAtomBytes, mk, &ctl->k_full[st], a * Cfg::kAtomE, ry, ti.hk, ti.kb);
#pragma unroll
      for (int a = 0; a < Cfg::kRAtoms; ++a)
        tma_load_4d(dst + (Cfg::kQAtoms + a) * Cfg::kAtomBytes, &p.tm_kr, &ctl->k_full[st],
                    a * Cfg::kAtomE, krow, ti.hk, ti.kb);
    }
    log.k_last[st] = static_cast<int32_t>(n);
    return true;
  };
  auto load_v = [&](const TileInfo &ti, int32_t j) -> bool {
    const uint32_t gg = g + j, st = gg % Cfg::kVStages, n = gg / Cfg::kVStages;
    if (!bwait_w(&ctl->v_empty[st], (n + 1) & 1, &ctl->abort, p)) return false;
    const int32_t krow = ti.krow + j * kBlockN;
    const bool fz = Cfg::kFuse && krow >= p.fuse_lo && krow < p.fuse_hi;
    const CUtensorMap *mv = fz ? &p.tm_vc : &p.tm_v;
    const int32_t ry = fz ? krow - p.fuse_lo : krow;
    uint8_t *dst = smem + Cfg::kVOff + st * Cfg::kVBytes;
    if (leader) {
      mbar_arrive_expect_tx(&ctl->v_full[st], Cfg::kVBytes);
#pragma unroll
      for (int a = 0; a < Cfg::kVAtoms; ++a)
        tma_load_4d(dst + a * Cfg::kAtomBytes, mv, &ctl->v_full[st], a * Cfg::kAtomE, ry, ti.hk, ti.kb);
    }
    log.v_last[st] = static_cast<int32_t>(n);
    return true;
  };

  for (uint32_t it = 0;; ++it) {
    // take the next item and publish it to the other roles
    const uint32_t k = it & 1;
    if (!(ok = bwait_w(&ctl->sched_empty[k], ((it >> 1) + 1) & 1, &ctl->abort, p))) break;
    int32_t t = 0;
    if (leader) t = atomicAdd(p.counters, 1);
    t = __shfl_sync(0xffffffffu, t, leader_lane);
    if (p.unit_major && t < n_units) t = unit_major_item(p, t);
    TileInfo t0, t1;
    if (t < n_units) {
      t0 = tile_info(p, t, 0);
      t1 = tile_info(p, t, 1);
    }
    if (leader) {
      ctl->sched_item[k] = t;
      if (t < n_units) {
        ctl->sched_ti[k][0] = t0;
        ctl->sched_ti[k][1] = t1;
      }
      mbar_arrive(&ctl->sched_full[k]);
    }
    if (t >= n_units) break;
    const int32_t n_max = max(t0.n_kv, t1.n_kv);
    if (n_max == 0) continue;
    if (!(ok = bwait_w(&ctl->q_empty, (u + 1) & 1, &ctl->abort, p))) break;
    if (leader) mbar_arrive_expect_tx(&ctl->q_full, Cfg::kQBytes);
    log.q_last = static_cast<int32_t>(u);
#pragma unroll
    for (int s = 0; s < 2 && leader; ++s) {
      const TileInfo &ts = s ? t1 : t0;
      uint8_t *qdst = smem + s * Cfg::kQTileBytes;
#pragma unroll
      for (int a = 0; a < Cfg::kQAtoms; ++a)
        tma_load_4d(qdst + a * Cfg::kAtomBytes, &p.tm_q, &ctl->q_full, a * Cfg::kAtomE, ts.qrow,
                    ts.h, ts.tma_b);
#pragma unroll
      for (int a = 0; a < Cfg::kRAtoms; ++a)
        tma_load_4d(qdst + (Cfg::kQAtoms + a) * Cfg::kAtomBytes, &p.tm_qr, &ctl->q_full,
                    a * Cfg::kAtomE, ts.qrow, ts.h, ts.tma_b);
    }
    // consumption order of the MMA thread: K0, then per j: V(j-1), K(j)...;
    // keep K one tile ahead of V.
    if (!(ok = load_k(t0, 0))) break;
    for (int32_t j = 0; j < n_max && ok; ++j) {
      if (j + 1 < n_max && !(ok = load_k(t0, j + 1))) break;
      ok = load_v(t0, j);
    }
    if (!ok) break;
    g += n_max;
    ++u;
  }
}

// ----------------------------------------------------------------------- MMA
// S = Q K^T: k-steps 0..KS, unrolled at compile time; q / k are the tile
// descriptors, each k-step moves both by the same compile-time offset.
template <typename Cfg, int KS>
struct IssueS {
  static __device__ __forceinline__ void run(uint32_t d, Desc q, Desc k) {
    if constexpr (KS > 0) IssueS<Cfg, KS - 1>::run(d, q, k);
    constexpr bool rope = KS >= Cfg::kSKStepsQK;
    constexpr int atom = rope ? Cfg::kQAtoms + (KS - Cfg::kSKStepsQK) / 4 : KS / 4;
    constexpr int within = (rope ? (KS - Cfg::kSKStepsQK) % 4 : KS % 4) * 32;
    constexpr int off = (atom * Cfg::kAtomBytes + within) >> 4;
    mma_f16_ss_at<off, off>(d, q, k, Cfg::kIdescS, KS > 0 ? 1u : 0u);
  }
};
// O (+)= P V: P read from TMEM (8 columns per k-step), V MN-major (16 rows of
// 128 bytes per k-step); k-steps K0..KS.
template <typename Cfg, int K0, int KS>
struct IssuePV {
  static __device__ __forceinline__ void run(uint32_t d, uint32_t p_tmem, Desc v, uint32_t acc0) {
    if constexpr (KS > K0) IssuePV<Cfg, K0, KS - 1>::run(d, p_tmem, v, acc0);
    mma_f16_ts_at<KS * 8, ((KS * Cfg::kKStep * 128) >> 4)>(d, p_tmem, v, Cfg::kIdescPV,
                                                         KS > 0 ? 1u : acc0);
  }
};

template <typename Cfg>
__device__ __forceinline__ void pp_issue_s(uint32_t tmem, Desc q, Desc k, int s) {
  IssueS<Cfg, Cfg::kSKStepsQK + Cfg::kSKStepsR - 1>::run(tmem + (s ? 128u : 0u), q, k);
}

// k-steps [K0, K1) of PV (keys 16 K0 .. 16 K1 of the tile).
template <typename Cfg, int K0, int K1>
__device__ __forceinline__ void pp_issue_pv(uint32_t tmem, Desc v, int s, bool accumulate) {
  if constexpr (K1 > K0)
    IssuePV<Cfg, K0, K1 - 1>::run(tmem + (s ? 384u : 256u), tmem + (s ? 128u : 0u), v,
                                  accumulate ? 1u : 0u);
}

template <typename Cfg>
__device__ void pp_mma(const AttnParams &p, uint8_t *smem, PPCtrl *ctl, uint32_t tmem, bool leader) {
  const int32_t n_units = num_units(p);
  uint32_t g = 0, u = 0;
  uint32_t cp[2] = {0, 0};    // PVs issued per tile slot (p_full completions consumed)
  uint32_t co[2] = {0, 0};    // units in which each tile slot took part (o_empty phases)
  bool ok = true;
  // descriptor bases, computed once: Q tiles, and stage 0 of the K / V rings
  // (stage i adds i * bytes-per-stage >> 4 to the low word)
  const Desc qb[2] = {desc_split(smem_desc_sw128(smem_u32(smem), 16, 1024)),
                      desc_split(smem_desc_sw128(smem_u32(smem + Cfg::kQTileBytes), 16, 1024))};
  const Desc k0 = desc_split(smem_desc_sw128(smem_u32(smem + Cfg::kKOff), 16, 1024));
  const Desc v0 = desc_split(smem_desc_sw128(smem_u32(smem + Cfg::kVOff), Cfg::kAtomBytes, 1024));
  auto kbase = [&](uint32_t gg) {
    return Desc{k0.lo + (gg % Cfg::kKStages) * (Cfg::kKBytes >> 4), k0.hi};
  };
  auto vbase = [&](uint32_t gg) {
    return Desc{v0.lo + (gg % Cfg::kVStages) * (Cfg::kVBytes >> 4), v0.hi};
  };
  auto wait_k = [&](uint32_t gg) {
    return bwait_w(&ctl->k_full[gg % Cfg::kKStages], (gg / Cfg::kKStages) & 1, &ctl->abort, p);
  };
  auto wait_v = [&](uint32_t gg) {
    return bwait_w(&ctl->v_full[gg % Cfg::kVStages], (gg / Cfg::kVStages) & 1, &ctl->abort, p);
  };
  // Fused cache write: the CTAs of the first unit of each kv head store the
  // new chunk's K / V tiles from shared memory into the cache as soon as they
  // have landed; each stage is released only after its store has read it.
  TileInfo ti0{};
  bool writer = false, pending = false;
  auto store_tile = [&](bool is_k, uint32_t gg, int32_t jj) {
    if constexpr (!Cfg::kFuse) return;
    const int32_t krow = ti0.krow + jj * kBlockN;
    if (!leader || !writer || krow < p.fuse_lo || krow >= p.fuse_hi) return;
    fence_proxy_async();
    const uint8_t *src = is_k ? smem + Cfg::kKOff + (gg % Cfg::kKStages) * Cfg::kKBytes
                              : smem + Cfg::kVOff + (gg % Cfg::kVStages) * Cfg::kVBytes;
    const int atoms = is_k ? Cfg::kQAtoms : Cfg::kVAtoms;
    for (int a = 0; a < atoms; ++a)
      tma_store_4d(is_k ? &p.tm_k : &p.tm_v, src + a * Cfg::kAtomBytes, a * Cfg::kAtomE, krow, ti0.hk,
                   ti0.kb);
    bulk_commit_group();
    pending = true;
  };
  auto stores_read = [&]() {
    if (Cfg::kFuse && pending && leader) {
      bulk_wait_read();
      pending = false;
    }
  };
  // PV of tile slot s for KV tile (unit-local) jj; returns false on abort.
  auto do_pv = [&](int s, int32_t jj, int32_t n_s, uint32_t gg) -> bool {
    constexpr int kSplitSteps = Cfg::kPSplit / Cfg::kKStep;
    if (jj == 0 && !bwait_w(&ctl->o_empty[s], (co[s] + 1) & 1, &ctl->abort, p)) return false;
    if constexpr (kSplitSteps > 0) {
      if (!bwait_w(&ctl->p_part[s], cp[s] & 1, &ctl->abort, p)) return false;
      tc_fence_after();
      if (leader) pp_issue_pv<Cfg, 0, kSplitSteps>(tmem, vbase(gg), s, jj > 0);
    }
    if (!bwait_w(&ctl->p_full[s], cp[s] & 1, &ctl->abort, p)) return false;
    tc_fence_after();
    if (leader) pp_issue_pv<Cfg, kSplitSteps, Cfg::kPVKSteps>(tmem, vbase(gg), s, jj > 0);
    ++cp[s];
    if (jj == n_s - 1 && leader) tc_commit(&ctl->o_full[s]);
    return true;
  };

  // Early start of tile A: when tile B has steps left after tile A's last PV
  // of an item (the causal diagonal), the next item is taken from the ring
  // right away and, once its Q and first K tile are in, its S_A(0) is issued
  // before B's last P is waited for, so tile A's softmax starts the next item
  // as soon as its epilogue is done instead of idling through B's extra step
  // (clock64 trace of the causal GQA prefill at B 4, 32/8 heads, L 4096:
  // ~6 400 cycles a boundary; +1.6% there).  `taken`: the
  // next item is in t_next / tis_next; `early`: its Q and K0 were waited for
  // and its S_A(0) issued.  Not in the fused instance, whose stores follow the
  // item, nor with a rope part: that S product is 1.5 times longer, and ahead
  // of B's last PV it delayed B by more than A gained (MLA -1.6%).
  bool taken = false, early = false, last = false;
  int32_t t_next = 0;
  TileInfo tis_next[2] = {};
  for (uint32_t it = 0;;) {
    int32_t t;
    TileInfo tis[2];
    const bool pre = early;
    if (taken) {
      t = t_next;
      tis[0] = tis_next[0];
      tis[1] = tis_next[1];
      taken = early = false;
    } else if (!(ok = pp_next_item(p, ctl, it, t, tis, -1, leader)) || t >= n_units) {
      break;
    }
    ti0 = tis[0];
    const int32_t n[2] = {tis[0].n_kv, tis[1].n_kv};
    const int32_t n_max = max(n[0], n[1]);
    if (n_max == 0) continue;
    writer = Cfg::kFuse && ti0.q0 == 0 && ti0.h % p.group == 0;
    if (!pre) {
      if (!(ok = bwait_w(&ctl->q_full, u & 1, &ctl->abort, p))) break;
      if (!(ok = wait_k(g))) break;
      tc_fence_after();
      store_tile(true, g, 0);
    }
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      if (n[s] > 0 && leader && !(pre && s == 0)) {
        pp_issue_s<Cfg>(tmem, qb[s], kbase(g), s);
        tc_commit(&ctl->s_full[s]);
      }
    }
    stores_read();
    if (leader) tc_commit(&ctl->k_empty[g % Cfg::kKStages]);
    for (int32_t j = 1; j < n_max && ok; ++j) {
      const uint32_t gk = g + j, gv = g + j - 1;
      if (!(ok = wait_k(gk))) break;
      store_tile(true, gk, j);
      if (!(ok = wait_v(gv))) break;
      store_tile(false, gv, j - 1);
      if (j - 1 < n[0] && !(ok = do_pv(0, j - 1, n[0], gv))) break;
      if (j < n[0] && leader) {
        pp_issue_s<Cfg>(tmem, qb[0], kbase(gk), 0);
        tc_commit(&ctl->s_full[0]);
      }
      if (j - 1 < n[1] && !(ok = do_pv(1, j - 1, n[1], gv))) break;
      stores_read();
      // With a single V stage (MLA tiles) V(j-1), now handed to both PVs, is
      // released before S_B(j) is issued, so that the next V load starts one
      // S product earlier (the commit still completes only once the PVs have);
      // with two stages the extra commit on this path costs more than it buys.
      if constexpr (Cfg::kVStages == 1)
        if (leader) tc_commit(&ctl->v_empty[gv % Cfg::kVStages]);
      if (j < n[1] && leader) {
        pp_issue_s<Cfg>(tmem, qb[1], kbase(gk), 1);
        tc_commit(&ctl->s_full[1]);
      }
      if (leader) tc_commit(&ctl->k_empty[gk % Cfg::kKStages]);
      if constexpr (Cfg::kVStages != 1)
        if (leader) tc_commit(&ctl->v_empty[gv % Cfg::kVStages]);
    }
    if (!ok) break;
    // All S products of this unit are issued: Q may be replaced once they finish.
    if (leader) tc_commit(&ctl->q_empty);
    if constexpr (!Cfg::kFuse && Cfg::kRAtoms == 0) {
      if (n[0] < n_max) {
        if (!(ok = pp_next_item(p, ctl, it, t_next, tis_next, -1, leader))) break;
        taken = t_next < n_units;
        last = !taken;
        if (taken && tis_next[0].n_kv > 0) {    // then the producer loads its Q
          const uint32_t g2 = g + n_max;
          if (!(ok = bwait_w(&ctl->q_full, (u + 1) & 1, &ctl->abort, p))) break;
          if (!(ok = wait_k(g2))) break;
          tc_fence_after();
          if (leader) {
            pp_issue_s<Cfg>(tmem, qb[0], kbase(g2), 0);
            tc_commit(&ctl->s_full[0]);
          }
          early = true;
        }
      }
    }
    const uint32_t gl = g + n_max - 1;
    if (!(ok = wait_v(gl))) break;
    store_tile(false, gl, n_max - 1);
#pragma unroll
    for (int s = 0; s < 2; ++s)
      if (n_max - 1 < n[s] && !(ok = do_pv(s, n_max - 1, n[s], gl))) break;
    if (!ok) break;
    stores_read();
    if (leader) tc_commit(&ctl->v_empty[gl % Cfg::kVStages]);
    for (int s = 0; s < 2; ++s)
      if (n[s] > 0) ++co[s];
    g += n_max;
    ++u;
    if (last) break;                  // the ring's end marker was taken early
  }
  if constexpr (Cfg::kFuse)
    if (leader) bulk_wait_all();   // cache stores complete before the CTA ends
  if (leader) tc_commit(&ctl->drain);
  drain_wait(&ctl->drain, 0, p);
}

// ------------------------------------------------------------------- softmax
// Epilogue through shared memory (p.tma_out, dense, no split): the warp's 32
// rows of O / l, each row in two 64-column halves, written as 16-bit pairs
// into its 4 KB staging area in the 128-byte swizzle of the output map and
// stored by one lane with a TMA tensor store (rows past Lq are clipped by the
// map).  With one thread per row, direct stores make every warp store
// instruction touch 32 rows (~1 000 store transactions per tile and item on
// the softmax warps' path); a half-row box is 4 KB in one bulk copy.
template <typename T, int DV>
__device__ __forceinline__ void store_rows_tma(const AttnParams &p, const TileInfo &ti, uint8_t *stage,
                                               const float (&o)[DV], float inv, int32_t row0) {
  static_assert(DV == 128, "two 64-column halves");
  const int lane = threadIdx.x & 31;
  const uint32_t base = smem_u32(stage) + lane * 128u;
#pragma unroll
  for (int hf = 0; hf < 2; ++hf) {
    if (lane == 0) bulk_wait_read();            // the area is free again (previous store read it)
    __syncwarp();
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const float *v = o + hf * 64 + c * 8;
      const uint32_t w0 = Elem16<T>::pack2(v[0] * inv, v[1] * inv), w1 = Elem16<T>::pack2(v[2] * inv, v[3] * inv);
      const uint32_t w2 = Elem16<T>::pack2(v[4] * inv, v[5] * inv), w3 = Elem16<T>::pack2(v[6] * inv, v[7] * inv);
      asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(base + ((c ^ (lane & 7)) << 4)), "r"(w0),
                   "r"(w1), "r"(w2), "r"(w3)
                   : "memory");
    }
    fence_proxy_async();
    __syncwarp();
    if (lane == 0) {
      tma_store_4d(&p.tm_o, stage, hf * 64, row0, ti.h, ti.b);
      bulk_commit_group();
    }
  }
}

// The same for split-KV partial rows (p.tma_part, dense): fp32 O / l of the
// split in four 32-column quarters (128 bytes of each row), stored into
// part_o at row part_rows index r0 (the warp's first row) and split `sp`.
// Only for warps whose 32 rows all lie below Lq: the partial rows of one
// (batch, head) are followed by the next head's.
template <int DV>
__device__ __forceinline__ void store_part_rows_tma(const AttnParams &p, uint8_t *stage, const float (&o)[DV],
                                                    float inv, int64_t r0, int32_t sp) {
  static_assert(DV == 128, "four 32-column quarters");
  const int lane = threadIdx.x & 31;
  const uint32_t base = smem_u32(stage) + lane * 128u;
#pragma unroll
  for (int qt = 0; qt < 4; ++qt) {
    if (lane == 0) bulk_wait_read();
    __syncwarp();
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const float *v = o + qt * 32 + c * 4;
      asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(base + ((c ^ (lane & 7)) << 4)),
                   "f"(v[0] * inv), "f"(v[1] * inv), "f"(v[2] * inv), "f"(v[3] * inv)
                   : "memory");
    }
    fence_proxy_async();
    __syncwarp();
    if (lane == 0) {
      tma_store_4d(&p.tm_po, stage, qt * 32, static_cast<int32_t>(r0), sp, 0);
      bulk_commit_group();
    }
  }
}

template <typename T, int DV, int kEmuPer16, bool kExplicit, bool kTmaEpi, int kPSplit>
__device__ void pp_softmax(const AttnParams &p, PPCtrl *ctl, uint32_t tmem, int s, uint8_t *stage) {
  const int32_t warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int32_t r = threadIdx.x & 127;                  // row within the tile = TMEM lane
  const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
  const uint32_t s_addr = tmem + lane_base + (s ? 128u : 0u);
  const uint32_t o_addr = tmem + lane_base + (s ? 384u : 256u);
  const int32_t n_units = num_units(p);
  uint32_t cs = 0, co = 0;
  bool ok = true;
  for (uint32_t it = 0;;) {
    int32_t t;
    TileInfo ti;
    ok = pp_next_item(p, ctl, it, t, &ti, s, false);
    __syncwarp();
    if (lane == 0 && ok) mbar_arrive(&ctl->sched_empty[(it - 1) & 1]);
    if (!ok || t >= n_units) break;
    const int32_t row = ti.q0 + r;
    const bool row_valid = row < ti.lq;
    if (ti.n_kv == 0) {
      if (row_valid) store_zero_row<T, DV>(p, ti, row);
      continue;
    }
    float m = -INFINITY, l = 0.f;
    for (int32_t j = 0; j < ti.n_kv; ++j) {
      if (!(ok = bwait(&ctl->s_full[s], cs & 1, &ctl->abort, p))) break;
      ++cs;
      tc_fence_after();
      uint32_t sr[128];
      tmem_ld_x128(s_addr, sr);
      float x[128];
      // S_s(j) done implies PV_s(j-1) done: O_s may be rescaled right away,
      // before any part of P_s(j) is handed to PV_s(j).
      auto first_part = [&](float a) {
        tmem_store_p_part<T, 0, kPSplit>(s_addr, x);
        if (j > 0 && __any_sync(0xffffffffu, a != 1.f)) tmem_scale_row<DV>(o_addr, a);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl->p_part[s]);
      };
      const float alpha = softmax_row<kEmuPer16, kExplicit, kPSplit>(p, ti, row, (ti.kt0 + j) * kBlockN,
                                                                     sr, x, m, l, first_part);
      tmem_store_p_part<T, kPSplit, 128>(s_addr, x);
      if (kPSplit == 0 && j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) tmem_scale_row<DV>(o_addr, alpha);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->p_full[s]);
    }
    if (!ok) break;
    if (!(ok = bwait(&ctl->o_full[s], co & 1, &ctl->abort, p))) break;
    ++co;
    tc_fence_after();
    float o[DV];
    tmem_load_row<DV>(o_addr, o);
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&ctl->o_empty[s]);
    if constexpr (kTmaEpi) {
      if (p.tma_out) {
        const float inv = l > 0.f ? 1.f / l : 0.f;
        store_rows_tma<T, DV>(p, ti, stage, o, inv, ti.q0 + (warp & 3) * 32);
        if (row_valid && p.lse)
          p.lse[(int64_t)ti.b * p.l_sb + (int64_t)ti.h * p.l_sh + (int64_t)row * p.l_si] =
              l > 0.f ? (m + __log2f(l)) * kLn2 : -INFINITY;
        continue;
      }
      const int32_t row0 = ti.q0 + (warp & 3) * 32;
      if (p.tma_part && p.n_split > 1 && !p.varlen && row0 + 32 <= ti.lq) {
        const int64_t r0 = ((int64_t)ti.b * p.hq + ti.h) * p.lq + row0;
        store_part_rows_tma<DV>(p, stage, o, l > 0.f ? 1.f / l : 0.f, r0, ti.sp);
        p.part_lse[(int64_t)ti.sp * p.part_rows + r0 + (r & 31)] =
            l > 0.f ? (m + __log2f(l)) * kLn2 : -INFINITY;
        continue;
      }
    }
    if (row_valid) store_result<T, DV>(p, ti, row, o, m, l);
  }
  if constexpr (kTmaEpi)
    if (lane == 0) bulk_wait_all();               // the output stores are done before the CTA ends
}

// --------------------------------------------------------------------- kernel
template <typename T, int DQK, int DROPE, int DV, int kKind>
__global__ void __launch_bounds__(kPPThreads, 1) attn_fwd_pp_kernel(const __grid_constant__ AttnParams p) {
  using Cfg = PPCfg<T, DQK, DROPE, DV, kKind>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  PPCtrl *ctl = reinterpret_cast<PPCtrl *>(smem + Cfg::kCtrlOff);
  const int32_t warp = threadIdx.x >> 5;

  if (threadIdx.x == 0) {
    mbar_init(&ctl->q_full, 1);
    mbar_init(&ctl->q_empty, 1);
    mbar_init(&ctl->drain, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&ctl->s_full[i], 1);
      mbar_init(&ctl->p_part[i], 4);
      mbar_init(&ctl->p_full[i], 4);
      mbar_init(&ctl->o_full[i], 1);
      mbar_init(&ctl->o_empty[i], 4);
    }
    for (int i = 0; i < 3; ++i) {
      mbar_init(&ctl->k_full[i], 1);
      mbar_init(&ctl->k_empty[i], 1);
      mbar_init(&ctl->v_full[i], 1);
      mbar_init(&ctl->v_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&ctl->sched_full[i], 1);
      mbar_init(&ctl->sched_empty[i], kSchedConsumers);
    }
    ctl->abort = 0;
    mbar_fence_init();
  }
  if (warp == 9) {
    tmem_alloc(&ctl->tmem_base, Cfg::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;
  pdl_wait();                       // the previous launch's results are visible from here on

  ProducerLog plog;
  if (warp < 8) {
    regs_increase<kPPSoftmaxRegs>();
    pp_softmax<T, DV, Cfg::kEmuPer16, Cfg::kMask, Cfg::kTmaEpi, Cfg::kPSplit>(p, ctl, tmem, warp >> 2,
                                                                smem + Cfg::kStageOff + warp * 4096);
  } else {
    regs_decrease<kPPOtherRegs>();
    if (warp == 8) pp_producer<Cfg>(p, smem, ctl, plog, elect_one());
    if (warp == 9) pp_mma<Cfg>(p, smem, ctl, tmem, elect_one());
  }
  pdl_trigger();

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, Cfg::kTmemCols);
  } else if (warp == 8 && (threadIdx.x & 31) == 0) {
    if (plog.q_last >= 0) drain_wait(&ctl->q_full, plog.q_last & 1, p);
    for (int s = 0; s < Cfg::kKStages; ++s)
      if (plog.k_last[s] >= 0) drain_wait(&ctl->k_full[s], plog.k_last[s] & 1, p);
    for (int s = 0; s < Cfg::kVStages; ++s)
      if (plog.v_last[s] >= 0) drain_wait(&ctl->v_full[s], plog.v_last[s] & 1, p);
    // Every fetch of this CTA has returned; the last CTA out resets the
    // item counter and the exit count for the next launch.
    __threadfence();
    if (atomicAdd(p.counters + 1, 1) == static_cast<int32_t>(gridDim.x) - 1) {
      atomicExch(p.counters, 0);
      atomicExch(p.counters + 1, 0);
    }
  }
}

template <typename T, int DQK, int DROPE, int DV, int kKind>
cudaError_t launch_attn_pp(const AttnParams &p, int grid, cudaStream_t stream) {
  using Cfg = PPCfg<T, DQK, DROPE, DV, kKind>;
  auto kern = attn_fwd_pp_kernel<T, DQK, DROPE, DV, kKind>;
  static SmemLimitRecord limit;       // this kernel's
  cudaError_t e = limit.ensure(kern, Cfg::kSmemBytes);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3(grid), dim3(kPPThreads), Cfg::kSmemBytes, stream, p);
}

}  // namespace wf
