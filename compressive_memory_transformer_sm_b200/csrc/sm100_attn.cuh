// attn_tc_kernel: A_dot (Eq. 6) + A_mem (Eq. 7) + gate (Eq. 10) of the
// Infini-attention forward, fused, on the sm_100a tensor cores: a persistent
// kernel whose work items are (b, h, segment, pair of 128-row query tiles).
#pragma once

#include "sm100_common.cuh"

namespace infini {
namespace tc {

// Pipeline timestamps of one CTA (block INFINI_ATTN_TRACE) for tuning builds:
// item `it` of softmax warpgroup k at 1024 * k + 16 * it + event, of the MMA
// thread at 2048 + 16 * it + event, of the TMA thread at 3072 + 16 * it +
// event; kernel start / setup done at 4000 / 4001.  Compiled out unless
// INFINI_ATTN_TRACE is defined.
#ifdef INFINI_ATTN_TRACE
__device__ unsigned long long g_attn_trace[4096];
#define ATTN_TRACE_VAL(cond, slot, val)                                                           \
  do {                                                                                            \
    if ((cond) && blockIdx.x == INFINI_ATTN_TRACE && (slot) < 4096) g_attn_trace[(slot)] = (val); \
  } while (0)
#else
#define ATTN_TRACE_VAL(cond, slot, val) \
  do {                                  \
  } while (0)
#endif
#define ATTN_TRACE(cond, slot) ATTN_TRACE_VAL(cond, slot, clock64())

struct AttnArgs {
  const float* beta;
  const float* snapz;     // [BH][S][128] fp32: z_{s-1}
  __nv_bfloat16* out;
  unsigned int* work_counter;  // next unclaimed work item; zero at launch (items < 2^31)
  int B, H, S, T;         // T = query tiles per full segment
  int P;                  // work items per full segment: ceil(T / 2) pairs, or T tiles (modes 1, 2)
  int GS;                 // segments per scheduling group
  // 0: a pair of query tiles per work item; 1: one query tile per item,
  // warpgroup 1 idle; 2: one query tile per item, its key tiles split between
  // the two warpgroups and their softmax states merged (small grids)
  int single;
  long long L;
  int N;
  float scale_log2;       // softmax scale * log2(e)
  long long os[3];        // element strides of out
  // Un-rotated q for sigma(Q) when the Q tiles loaded by TMA carry rotary
  // position embeddings (local attention only); nullptr: sigma(Q) from the
  // Q tiles themselves.  qms: element strides of its (B, H, L) dimensions.
  const __nv_bfloat16* qm;
  long long qms[3];
  // For the backward's recomputation (nullptr otherwise): A_dot of every row
  // in fp32, contiguous [B*H*L][128], and the row's log2-sum-exp2 of the
  // scaled scores (P = 2^(s * scale_log2 - lse2)), [B*H*L] fp32.
  float* adot;
  float* lse2;
};

// Shared memory of the attention kernel (offsets from a 1024-aligned base).
constexpr int kKStages = 3;          // K ring depth (V ring: 2)
constexpr int kItemSlots = 2;        // work items handed from the TMA thread to the consumers
constexpr uint32_t kA_Q0 = 0;
constexpr uint32_t kA_Q1 = 32768;
constexpr uint32_t kA_K0 = 65536;    // K ring: 3 stages of 32 KB
constexpr uint32_t kA_V0 = kA_K0 + kKStages * 32768u;  // V ring: 2 stages of 32 KB
constexpr uint32_t kA_Z = kA_V0 + 2 * 32768u;  // z_{s-1}, one copy per softmax warpgroup
constexpr uint32_t kA_BAR = kA_Z + 1024;
constexpr int kAttnThreads = 384;
// Register split: the kernel launches with 168 registers per thread (384 x 168
// = 64512); the load/MMA warpgroup gives back to 88 and the two softmax
// warpgroups take 208: 2 x 128 x 208 + 128 x 88 = 64512 (the split with no
// spills on either side).  The build checks
// that ptxas allocated exactly kAttnLaunchRegs, else an increase could wait
// forever.
constexpr uint32_t kAttnLaunchRegs = 168, kAttnSoftmaxRegs = 208, kAttnOtherRegs = 88;
static_assert(2 * 128 * kAttnSoftmaxRegs + 128 * kAttnOtherRegs == kAttnThreads * kAttnLaunchRegs,
              "register split must add up to the launch allocation");

// Barrier indices.
enum : int {
  B_Q = 0,
  B_KF0 = 1,   // K stage full (2)
  B_VF0 = 3,   // V stage full (2)
  B_KE0 = 5,   // K stage free: both S products of that key tile done (2)
  B_SF0 = 7,   // S of query tile k ready (2)
  B_PF0 = 9,   // P of query tile k written (2, 128 arrivals)
  B_SQ0 = 11,  // sigma(Q) of query tile k written (2, 128 arrivals)
  B_MEM0 = 13, // sigma(Q_k) M_{s-1} ready (2)
  B_VE0 = 15,  // V stage free: both P V products of that key tile done (2)
  B_KF2 = 17,  // third K stage full
  B_KE2 = 18,  // third K stage free
  B_OF0 = 19,  // TMEM S_k / O_k read out by the epilogue of query tile k (2, 128 arrivals)
  B_IF0 = 21,  // work-item slot published (kItemSlots)
  B_IE0 = 23,  // work-item slot read by every consumer (kItemSlots)
  B_DONE = 25, // every product issued by the MMA thread complete (exit)
  B_PH0 = 26,  // first half of P (keys 0-63) of query tile k written (2, 128 arrivals)
  B_COUNT = 28
};
constexpr uint32_t kA_ITEMS = kA_BAR + 8 * B_COUNT;  // kItemSlots x int64 work-item indices
constexpr uint32_t kA_TMEMSLOT = kA_ITEMS + 8 * kItemSlots;
constexpr uint32_t kAttnSmem = kA_TMEMSLOT + 16 + 1024;  // + alignment slack
static_assert(kAttnSmem <= 232448, "attention kernel exceeds 227 KB of shared memory");

// Persistent kernel, one CTA per SM.  A work item is two adjacent 128-row
// query tiles (2m, 2m+1) of one (b, h, segment), sharing every K/V tile load
// between them (or the single tile m when `single`).  The TMA thread claims
// items from a global counter in the grouped order below and hands each to
// the other roles through a two-slot ring in shared memory; every role keeps
// running barrier phases across the CTA's items, so the loads and the first
// products of the next item overlap the epilogue of the current one.
//
// Warps 0-3: softmax warpgroup of query tile 2m; warps 4-7: of tile 2m+1
// (thread = query row = TMEM lane).  Warp 8 loads (TMA), warp 9 issues the
// MMAs and owns TMEM, warps 10-11 only complete their warpgroup.  TMEM columns: S of tile 2m [0,128), S of tile 2m+1
// [128,256), O of tile 2m [256,384), O of tile 2m+1 [384,512).  P (bf16)
// overwrites the first 64 columns of its S buffer and feeds the P V product
// from TMEM; after the last P V product the S buffer receives sigma(Q) M_{s-1}.
//
// MMA issue order (k = query tile): S_0(0) S_1(0) | PV_0(j-1) S_0(j) PV_1(j-1)
// S_1(j) | ... : the strict alternation keeps the two softmax warpgroups half
// a period apart, so one works while the tensor cores serve the other, and
// "S_k(j) complete" implies "PV_k(j-1) complete": the O rescale of the
// softmax needs no extra wait.
//
// Items are ordered by groups of GS segments (about one wave of items per
// group, so the group's K/V stays in L2), heaviest pair first inside a group;
// claiming them dynamically balances the CTAs.
// kSplit: the split schedule (a.single == 2), compiled as its own kernel so
// that the pair and single-tile schedules keep their code unchanged.
template <bool kSplit>
__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_mt,
                   const AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  ATTN_TRACE(threadIdx.x == 0, 4000);

  const int NS = a.B * a.H * a.S;
  const int per_group = a.GS * a.P;
  const int total = ((NS + a.GS - 1) / a.GS) * per_group;  // the host keeps this below 2^31
  const bool single = !kSplit && a.single == 1;
  constexpr bool split = kSplit;
  // Work item idx of the grouped heavy-first order -> (m, segment); false for
  // the padding of the last group and for tiles past the end of a short
  // (tail) segment.
  struct Item {
    int m, seg, b, h, n_s, tq0, nk0, nk1;
    long long seg0;
  };
  auto decode = [&](int idx, Item& it) -> bool {
    const int grp = idx / per_group;
    const int r = idx - grp * per_group;
    const int gsz = min(a.GS, NS - grp * a.GS);
    if (r >= gsz * a.P) return false;
    it.m = a.P - 1 - r / gsz;  // pair index, or tile index (modes 1, 2)
    it.seg = grp * a.GS + r % gsz;  // = bh * S + s
    const int bh = it.seg / a.S, s = it.seg % a.S;
    it.b = bh / a.H;
    it.h = bh % a.H;
    it.seg0 = (long long)s * a.N;
    it.n_s = (int)min((long long)a.N, a.L - it.seg0);
    it.tq0 = single || split ? it.m : 2 * it.m;  // query tile of warpgroup 0 (pairs: warpgroup 1 has tq0 + 1)
    if (split) {  // key tiles [0, nk0) to warpgroup 0, [nk0, nk0 + nk1) (with the diagonal) to warpgroup 1
      it.nk0 = (it.tq0 + 1) / 2;
      it.nk1 = it.tq0 + 1 - it.nk0;
    } else {
      it.nk0 = it.tq0 + 1;                    // K/V tiles of query tile tq0
      it.nk1 = it.tq0 + (single ? 1 : 2);     // K/V tiles of the item's last query tile
    }
    return it.tq0 * kTile < it.n_s;
  };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto sQ = [&](int k) { return base + (k ? kA_Q1 : kA_Q0); };
  auto sK = [&](int st) { return base + kA_K0 + (uint32_t)st * kTileBytes; };
  auto sV = [&](int st) { return base + kA_V0 + (uint32_t)st * kTileBytes; };
  auto bar = [&](int i) { return base + kA_BAR + 8u * (uint32_t)i; };
  // The K ring is used in order: every item's K tiles, then its M_{s-1}
  // snapshot.  Slot g (counted modulo 6 over all the CTA's items) lives in
  // stage g % 3, and its barriers (full / free) complete a phase of parity
  // g / 3 for it.  V-ring slot g (counted modulo 2^32): stage g % 2, parity
  // (g / 2) % 2.  A producer waits for the free phase of the previous use,
  // parity ^ 1, which a fresh barrier reports complete.
  auto knext = [](uint32_t g, int j) { return (g + (uint32_t)(j % 6)) % 6u; };
  auto kfull = [&](uint32_t g) { const uint32_t st = g % 3u; return bar(st < 2 ? B_KF0 + (int)st : B_KF2); };
  auto kfree = [&](uint32_t g) { const uint32_t st = g % 3u; return bar(st < 2 ? B_KE0 + (int)st : B_KE2); };
  auto kph = [](uint32_t g) { return g / 3u; };
  auto sKt = [&](uint32_t g) { return sK((int)(g % 3u)); };
  auto vfull = [&](uint32_t g) { return bar(B_VF0 + (int)(g & 1u)); };
  auto vfree = [&](uint32_t g) { return bar(B_VE0 + (int)(g & 1u)); };
  auto vph = [](uint32_t g) { return (g >> 1) & 1u; };
  auto sVt = [&](uint32_t g) { return sV((int)(g & 1u)); };
  float* zs = reinterpret_cast<float*>(gbase + kA_Z);
  int* slots = reinterpret_cast<int*>(gbase + kA_ITEMS);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + kA_TMEMSLOT);

  if (threadIdx.x == 0) {
    mbar_init(bar(B_Q), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(B_KF0 + i), 1);
      mbar_init(bar(B_VF0 + i), 1);
      mbar_init(bar(B_KE0 + i), 1);
      mbar_init(bar(B_VE0 + i), 1);
      mbar_init(bar(B_SF0 + i), 1);
      mbar_init(bar(B_PF0 + i), 128);
      mbar_init(bar(B_PH0 + i), 128);
      mbar_init(bar(B_SQ0 + i), 128);
      mbar_init(bar(B_MEM0 + i), 1);
      mbar_init(bar(B_OF0 + i), 128);
    }
    mbar_init(bar(B_KF2), 1);
    mbar_init(bar(B_KE2), 1);
    mbar_init(bar(B_DONE), 1);
    for (int i = 0; i < kItemSlots; ++i) {
      mbar_init(bar(B_IF0 + i), 1);
      mbar_init(bar(B_IE0 + i), single ? 1 + 128 : 1 + 256);  // lane 0 of the MMA warp + the softmax threads
    }
    fence_barrier_init();
  }
  if (warp == 9) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // Launched as a programmatic dependent (after the snapshot of a streaming
  // step), the setup above overlaps the previous kernel; nothing it wrote
  // (the snapshots, the work counter) is read before this returns.
  griddep_wait();
  // The CTA owns all 512 columns of the SM's tensor memory, so its block
  // starts at lane 0, column 0 and every TMEM address below is a constant.
  if (*tmem_slot != 0u) {  // not expected: report and leave
    if (threadIdx.x == 0) atomicOr(&g_status, kStatusTimeout);
    if (warp == 9) tmem_dealloc(*tmem_slot, 512);
    return;
  }
  constexpr uint32_t tmem = 0;
  ATTN_TRACE(threadIdx.x == 0, 4001);

  // Consumers take work item `it` of this CTA from slot it % kItemSlots
  // (-1: no more work, or a wait on this device gave up).
  auto take_item = [&](int it, bool arrive) -> int {
    const int sl = it % kItemSlots;
    mbar_wait(bar(B_IF0 + sl), (uint32_t)((it / kItemSlots) & 1));
    const int idx = *reinterpret_cast<volatile int*>(&slots[sl]);
    if (arrive) mbar_arrive(bar(B_IE0 + sl));
    return device_aborted() ? -1 : idx;
  };

  if (warp >= 8) {
  regs_decrease<kAttnOtherRegs>();
  if (warp == 8) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      prefetch_tensormap(&tm_q);
      prefetch_tensormap(&tm_k);
      prefetch_tensormap(&tm_v);
      prefetch_tensormap(&tm_mt);
      uint32_t gk = 0, gv = 0, nq = 0;  // next K-ring slot (mod 6), next V-ring slot, Q pairs loaded
      uint32_t kn = 0, vn = 0;          // K / V fills issued, saturating at the ring depth
      for (int it = 0;; ++it) {
        int idx = total;
        Item w;
        if (!device_aborted()) {
          do {
            idx = (int)atomicAdd(a.work_counter, 1u);
          } while (idx < total && !decode(idx, w));
        }
        ATTN_TRACE(true, 3072 + 16 * it + 0);
        ATTN_TRACE_VAL(true, 3072 + 16 * it + 8, (unsigned long long)idx);
        const int sl = it % kItemSlots;
        if (!mbar_wait(bar(B_IE0 + sl), (uint32_t)(((it / kItemSlots) & 1) ^ 1))) break;
        slots[sl] = idx < total ? idx : -1;
        mbar_arrive(bar(B_IF0 + sl));  // release: the consumers see the slot once the phase completes
        ATTN_TRACE(true, 3072 + 16 * it + 1);
        if (idx >= total) break;
        // K tile j once the S products of the slot's previous use are done; V
        // tile j-1 likewise after its P V products (V trails K by one tile, so
        // a pending V never holds back the next K).  Q after the memory-read
        // products of the previous item, which read sigma(Q) from the Q
        // tiles: issued after K tile 0 of the new item.
        if (split) {
          // Key tiles of the two warpgroups interleaved in both rings: step j
          // loads warpgroup 0's tile j (j < nk0), then warpgroup 1's tile
          // nk0 + j (j < nk1); V trails K by one step.  One Q tile.
          for (int j = 0; j <= w.nk1; ++j) {
            for (int kq = 0; kq < 2; ++kq) {
              if (j >= (kq ? w.nk1 : w.nk0)) continue;
              const int lk = (int)(w.seg0 + (long long)(kq ? w.nk0 + j : j) * kTile);
              if (!mbar_wait(kfree(gk), kph(gk) ^ 1u)) goto done;
              mbar_expect_tx(kfull(gk), kTileBytes);
              tma_load_4d(sKt(gk), &tm_k, kfull(gk), 0, lk, w.h, w.b);
              tma_load_4d(sKt(gk) + kBox, &tm_k, kfull(gk), 64, lk, w.h, w.b);
              gk = knext(gk, 1);
              kn = min(kn + 1u, (uint32_t)kKStages);
            }
            if (j == 0) {
              const uint32_t prev = (uint32_t)(it & 1) ^ 1u;  // previous item's phase (fresh: complete)
              if (!mbar_wait(bar(B_MEM0), prev)) goto done;
              const int lq = (int)(w.seg0 + (long long)w.tq0 * kTile);
              mbar_expect_tx(bar(B_Q), kTileBytes);
              tma_load_4d(sQ(0), &tm_q, bar(B_Q), 0, lq, w.h, w.b);
              tma_load_4d(sQ(0) + kBox, &tm_q, bar(B_Q), 64, lq, w.h, w.b);
              ++nq;
            }
            if (j >= 1) {
              for (int kq = 0; kq < 2; ++kq) {
                if (j - 1 >= (kq ? w.nk1 : w.nk0)) continue;
                const int lk = (int)(w.seg0 + (long long)(kq ? w.nk0 + j - 1 : j - 1) * kTile);
                if (!mbar_wait(vfree(gv), vph(gv) ^ 1u)) goto done;
                mbar_expect_tx(vfull(gv), kTileBytes);
                tma_load_4d(sVt(gv), &tm_v, vfull(gv), 0, lk, w.h, w.b);
                tma_load_4d(sVt(gv) + kBox, &tm_v, vfull(gv), 64, lk, w.h, w.b);
                ++gv;
                vn = min(vn + 1u, 2u);
              }
            }
          }
        } else {
          for (int j = 0; j <= w.nk1; ++j) {
            if (j < w.nk1) {
              const int lk = (int)(w.seg0 + (long long)j * kTile);
              if (!mbar_wait(kfree(gk), kph(gk) ^ 1u)) goto done;
              mbar_expect_tx(kfull(gk), kTileBytes);
              tma_load_4d(sKt(gk), &tm_k, kfull(gk), 0, lk, w.h, w.b);
              tma_load_4d(sKt(gk) + kBox, &tm_k, kfull(gk), 64, lk, w.h, w.b);
              gk = knext(gk, 1);
              kn = min(kn + 1u, (uint32_t)kKStages);
            }
            if (j == 0) {
              const uint32_t prev = (uint32_t)(it & 1) ^ 1u;  // previous item's phase (fresh: complete)
              if (!mbar_wait(bar(B_MEM0), prev)) goto done;
              if (!single && !mbar_wait(bar(B_MEM0 + 1), prev)) goto done;
              const int lq = (int)(w.seg0 + (long long)w.tq0 * kTile);
              mbar_expect_tx(bar(B_Q), (single ? 1 : 2) * kTileBytes);
              tma_load_4d(sQ(0), &tm_q, bar(B_Q), 0, lq, w.h, w.b);
              tma_load_4d(sQ(0) + kBox, &tm_q, bar(B_Q), 64, lq, w.h, w.b);
              if (!single) {
                tma_load_4d(sQ(1), &tm_q, bar(B_Q), 0, lq + kTile, w.h, w.b);
                tma_load_4d(sQ(1) + kBox, &tm_q, bar(B_Q), 64, lq + kTile, w.h, w.b);
              }
              ++nq;
              ATTN_TRACE(true, 3072 + 16 * it + 2);
            }
            if (j >= 1) {
              const int lk = (int)(w.seg0 + (long long)(j - 1) * kTile);
              if (!mbar_wait(vfree(gv), vph(gv) ^ 1u)) goto done;
              mbar_expect_tx(vfull(gv), kTileBytes);
              tma_load_4d(sVt(gv), &tm_v, vfull(gv), 0, lk, w.h, w.b);
              tma_load_4d(sVt(gv) + kBox, &tm_v, vfull(gv), 64, lk, w.h, w.b);
              ++gv;
              vn = min(vn + 1u, 2u);
            }
          }
        }
        // M_{s-1} (bf16 snapshot, [dk][dv]) enters the K ring after the item's K tiles.
        if (!mbar_wait(kfree(gk), kph(gk) ^ 1u)) goto done;
        mbar_expect_tx(kfull(gk), kTileBytes);
        tma_load_2d(sKt(gk), &tm_mt, kfull(gk), 0, w.seg * 128);
        tma_load_2d(sKt(gk) + kBox, &tm_mt, kfull(gk), 64, w.seg * 128);
        ATTN_TRACE(true, 3072 + 16 * it + 3);
        gk = knext(gk, 1);
        kn = min(kn + 1u, (uint32_t)kKStages);
      }
    done:
      if (device_aborted()) {
        // a wait gave up: let the copies still in flight land before the CTA exits
        for (uint32_t i = 1; i <= kn; ++i) {
          const uint32_t g = knext(gk, 6 - (int)i);
          mbar_drain(kfull(g), kph(g));
        }
        for (uint32_t i = 1; i <= vn; ++i) mbar_drain(vfull(gv - i), vph(gv - i));
        if (nq > 0) mbar_drain(bar(B_Q), (nq - 1u) & 1u);
      }
    }
  } else if (warp == 9) {
    {
      // The whole warp runs the issue loop (uniform control flow); one elected
      // lane issues the MMAs and the commits.
      // ------------------------------------------------------------ MMA issuer
      // Per key tile j of query tile k: P_k(j) (bf16, TMEM columns 0-63)
      // feeds P V in two halves, the first while the softmax still computes
      // the second; S_k(j+1) overwrites those columns after the second.
      constexpr uint32_t idesc_kk = idesc_bf16(128, 128, 0, 0);
      constexpr uint32_t idesc_pv = idesc_bf16(128, 128, 0, 1);
      constexpr uint32_t idesc_mem = idesc_bf16(128, 128, 0, 1);
      uint32_t gk = 0, gv = 0;           // next K / V ring slot
      uint32_t nt0 = 0, nt1 = 0;         // P tiles of query tile 0 / 1 so far (PH / PF phases)
      for (int it = 0;; ++it) {
        const int idx = take_item(it, lane == 0);  // one arrival for the warp
        if (idx < 0) break;
        Item w;
        decode(idx, w);
        // the Q tile addresses are re-derived per item so that their
        // descriptors are not kept live across the whole loop
        const uint32_t q0 = opaque_u32(sQ(0));
        auto sQi = [&](int k) { return q0 + (k ? kA_Q1 - kA_Q0 : 0u); };
        // S_k(j) = Q_k K_j^T
        auto issue_s = [&](int k, uint32_t g) {
          const uint64_t da = kmajor_base(sQi(k)), db = kmajor_base(sKt(g));
          if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              mma_ss(tmem + (uint32_t)k * 128u, da + kmajor_step(kk), db + kmajor_step(kk), idesc_kk, kk > 0 ? 1u : 0u);
          }
          __syncwarp();
        };
        // O_k (+)= P_k V: K-steps [4h, 4h + 4) = keys [64h, 64h + 64)
        auto issue_pv_half = [&](int k, uint32_t g, int h, bool first) {
          const uint64_t db = mnmajor_base(sVt(g));
          if (elect_one()) {
#pragma unroll
            for (int kk = 4 * h; kk < 4 * h + 4; ++kk)
              mma_ts(tmem + 256u + (uint32_t)k * 128u, tmem + (uint32_t)k * 128u + (uint32_t)kk * 8u,
                     db + mnmajor_step(kk), idesc_pv, (!first || kk > 0) ? 1u : 0u);
          }
          __syncwarp();
        };
        auto commit = [&](uint32_t b) {
          if (elect_one()) mma_commit(b);
          __syncwarp();
        };
        if (split) {
          // One query tile (Q_0) for both warpgroups; warpgroup k's key tile j
          // sits at ring position kpos(k, j) of the item (the producer's order).
          const uint32_t prev = (uint32_t)(it & 1) ^ 1u;
          const int n0 = w.nk0, n1 = w.nk1;
          auto kpos = [&](int k, int j) { return k == 0 ? 2 * j : j + min(j + 1, n0); };
          auto issue_sq = [&](int k, uint32_t g) {  // S_k = Q_0 K^T
            const uint64_t da = kmajor_base(sQi(0)), db = kmajor_base(sKt(g));
            if (elect_one()) {
#pragma unroll
              for (int kk = 0; kk < 8; ++kk)
                mma_ss(tmem + (uint32_t)k * 128u, da + kmajor_step(kk), db + kmajor_step(kk), idesc_kk, kk > 0 ? 1u : 0u);
            }
            __syncwarp();
          };
          mbar_wait(bar(B_Q), (uint32_t)(it & 1));
#pragma unroll 1
          for (int k = 0; k < 2; ++k) {
            if ((k ? n1 : n0) == 0) continue;
            const uint32_t g = knext(gk, kpos(k, 0));
            mbar_wait(kfull(g), kph(g));
            mbar_wait(bar(B_OF0 + k), prev);  // S_k(0) overwrites what the previous epilogue reads
            tc_fence_after();
            issue_sq(k, g);
            commit(bar(B_SF0 + k));
            commit(kfree(g));
          }
          for (int j = 0; j < n1; ++j) {
#pragma unroll 1
            for (int k = 0; k < 2; ++k) {
              const int nk = k ? n1 : n0;
              if (j >= nk) continue;
              const uint32_t gvj = gv + (uint32_t)kpos(k, j);
              uint32_t& nt = k ? nt1 : nt0;
              mbar_wait(vfull(gvj), vph(gvj));
              mbar_wait(bar(B_PH0 + k), nt & 1u);
              tc_fence_after();
              issue_pv_half(k, gvj, 0, j == 0);
              mbar_wait(bar(B_PF0 + k), nt & 1u);
              ++nt;
              tc_fence_after();
              issue_pv_half(k, gvj, 1, j == 0);
              commit(vfree(gvj));
              if (j + 1 < nk) {
                const uint32_t gn = knext(gk, kpos(k, j + 1));
                mbar_wait(kfull(gn), kph(gn));
                issue_sq(k, gn);
                commit(bar(B_SF0 + k));
                commit(kfree(gn));
              }
            }
          }
          commit(bar(B_MEM0 + 1));  // every product of warpgroup 1 complete: its O is final
          // memory read of the tile: sigma(Q_0) M_{s-1} into S_0's columns
          const uint32_t gm = knext(gk, n0 + n1);
          mbar_wait(kfull(gm), kph(gm));
          mbar_wait(bar(B_OF0), prev);  // (no S_0 product waited for it when n0 = 0)
          mbar_wait(bar(B_SQ0), (uint32_t)(it & 1));
          tc_fence_after();
          {
            const uint64_t da = kmajor_base(sQi(0)), db = mnmajor_base(sKt(gm));
            if (elect_one()) {
#pragma unroll
              for (int kk = 0; kk < 8; ++kk)
                mma_ss(tmem, da + kmajor_step(kk), db + mnmajor_step(kk), idesc_mem, kk > 0 ? 1u : 0u);
            }
            __syncwarp();
          }
          commit(bar(B_MEM0));
          commit(kfree(gm));
          gk = knext(gm, 1);
          gv += (uint32_t)(n0 + n1);
          continue;
        }
        const uint32_t prev = (uint32_t)(it & 1) ^ 1u;  // previous item's phase (fresh: complete)
        ATTN_TRACE(true, 2048 + 16 * it + 0);
        mbar_wait(bar(B_Q), (uint32_t)(it & 1));
        ATTN_TRACE(true, 2048 + 16 * it + 1);
        mbar_wait(kfull(gk), kph(gk));
        // S_k(0) overwrites the S_k / O_k columns the previous item's epilogue reads
        mbar_wait(bar(B_OF0), prev);
        tc_fence_after();
        issue_s(0, gk);
        commit(bar(B_SF0));
        ATTN_TRACE(true, 2048 + 16 * it + 2);
        if (!single) {
          mbar_wait(bar(B_OF0 + 1), prev);
          tc_fence_after();
          issue_s(1, gk);
          commit(bar(B_SF0 + 1));
          ATTN_TRACE(true, 2048 + 16 * it + 3);
        }
        commit(kfree(gk));
        // one step per key tile j: the P V products of tile j and S(j + 1), query tile 0 then 1
        for (int j = 0; j < w.nk1; ++j) {
          const uint32_t gvj = gv + (uint32_t)j, gn = knext(gk, j + 1);
          const bool more = j + 1 < w.nk1;  // key tile j + 1 exists (for query tile 1)
          if (more) mbar_wait(kfull(gn), kph(gn));
          mbar_wait(vfull(gvj), vph(gvj));
#pragma unroll 1
          for (int k = 0; k < 2; ++k) {
            const int nk = k ? w.nk1 : w.nk0;  // key tiles of query tile k
            if ((k == 1 && single) || j >= nk) continue;
            const bool next = j + 1 < nk;
            uint32_t& nt = k ? nt1 : nt0;
            mbar_wait(bar(B_PH0 + k), nt & 1u);
            ATTN_TRACE(it == 0, 2560 + 8 * j + 3 * k + 1);
            tc_fence_after();
            issue_pv_half(k, gvj, 0, j == 0);
            mbar_wait(bar(B_PF0 + k), nt & 1u);
            ++nt;
            ATTN_TRACE(it == 0, 2560 + 8 * j + 3 * k + 2);
            tc_fence_after();
            issue_pv_half(k, gvj, 1, j == 0);
            if (next) {
              issue_s(k, gn);
              commit(bar(B_SF0 + k));
            }
          }
          commit(vfree(gvj));
          if (more) commit(kfree(gn));
        }
        ATTN_TRACE(true, 2048 + 16 * it + 4);
        // memory read: sigma(Q_k) (written over Q_k by the softmax warps) times M_{s-1}
        const uint32_t gm = knext(gk, w.nk1);
        mbar_wait(kfull(gm), kph(gm));
        const uint32_t mt = sKt(gm);  // M_{s-1} [dk][dv]: MN-major B operand (like V)
#pragma unroll 1
        for (int k = 0; k < (single ? 1 : 2); ++k) {
          mbar_wait(bar(B_SQ0 + k), (uint32_t)(it & 1));
          tc_fence_after();
          const uint64_t da = kmajor_base(sQi(k)), db = mnmajor_base(mt);
          if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              mma_ss(tmem + (uint32_t)k * 128u, da + kmajor_step(kk), db + mnmajor_step(kk), idesc_mem, kk > 0 ? 1u : 0u);
          }
          __syncwarp();
          commit(bar(B_MEM0 + k));
          ATTN_TRACE(true, 2048 + 16 * it + 5 + k);
        }
        commit(kfree(gm));
        gk = knext(gm, 1);
        gv += (uint32_t)w.nk1;
      }
      // every product issued has completed before TMEM is released
      if (elect_one()) {
        mma_commit(bar(B_DONE));
        mbar_drain(bar(B_DONE), 0);
      }
      __syncwarp();
    }
  }
  } else {
    regs_increase<kAttnSoftmaxRegs>();
    // -------------------------------------------------------------- softmax WGs
    const int k = warp >> 2;  // query tile tq0 + k of each item
    if (!(single && k == 1)) {
    const int row = (warp & 3) * 32 + lane;  // query row in the tile = TMEM lane
    const uint32_t lrow = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lrow + (uint32_t)k * 128u;
    const uint32_t tO = tmem + lrow + 256u + (uint32_t)k * 128u;
    const float c = a.scale_log2;
    const bool tr = (row == 0);
    uint32_t ns = 0;  // S tiles of query tile k so far (phase of its S barrier)
    for (int it = 0;; ++it) {
      const int idx = take_item(it, true);
      if (idx < 0) break;
      Item w;
      decode(idx, w);
      // its K/V tiles; the last one is its diagonal (split: warpgroup 1's last)
      const int nk = split ? (k ? w.nk1 : w.nk0) : w.nk0 + k;
      ATTN_TRACE(tr, 1024 * k + 16 * it + 0);
      ATTN_TRACE_VAL(tr, 1024 * k + 16 * it + 8, (unsigned long long)nk);
      const float zrow = a.snapz[(long long)w.seg * 128 + row];  // used after the loop
      float m_ref = 0.f, l = 0.f;
      for (int j = 0; j < nk; ++j) {
        mbar_wait(bar(B_SF0 + k), ns & 1u);
        ++ns;
        ATTN_TRACE(tr && j == 0, 1024 * k + 16 * it + 1);
        ATTN_TRACE(tr && it == 0, 1024 * k + 512 + 8 * j + 0);
        tc_fence_after();
        uint32_t x[128];
        {
          uint32_t (&x0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&x[0]);
          uint32_t (&x1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&x[32]);
          uint32_t (&x2)[32] = *reinterpret_cast<uint32_t(*)[32]>(&x[64]);
          uint32_t (&x3)[32] = *reinterpret_cast<uint32_t(*)[32]>(&x[96]);
          tmem_ld32(tS, x0);
          tmem_ld32(tS + 32u, x1);
          tmem_ld32(tS + 64u, x2);
          tmem_ld32(tS + 96u, x3);
          tmem_ld_wait();
        }
        ATTN_TRACE(tr && it == 0, 1024 * k + 512 + 8 * j + 2);
        if (j == nk - 1 && (!split || k == 1)) {  // diagonal tile: key e is visible to query row iff e <= row
#pragma unroll
          for (int e = 0; e < 128; ++e)
            if (e > row) x[e] = __float_as_uint(-INFINITY);
        }
        float mx[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) mx[i] = __uint_as_float(x[i]);
#pragma unroll
        for (int e = 4; e < 128; ++e) mx[e & 3] = fmaxf(mx[e & 3], __uint_as_float(x[e]));
        const float mxs = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * c;
        // Move the reference max only when the row max grows by more than 2^8:
        // O / l stays exact for any reference, and p stays below 256.
        const float m_new = (j == 0) ? mxs : (mxs > m_ref + 8.f ? mxs : m_ref);
        const bool resc = (j > 0) && (m_new != m_ref);
        if (__any_sync(0xffffffffu, resc)) {
          // S_k(j) complete implies P V of tile j-1 complete (issue order), so O is final here.
          const float alpha = resc ? ex2_approx(m_ref - m_new) : 1.f;
          l *= alpha;
          uint32_t o[16];
#pragma unroll 1
          for (int cc = 0; cc < 8; ++cc) {
            tmem_ld16(tO + 16u * cc, o);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            tmem_st16(tO + 16u * cc, o);
          }
          tmem_st_wait();
        }
        m_ref = m_new;
        const float nm = -m_ref;
        float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int e = 0; e < 64; ++e) {
          // scale-and-subtract and the row sum in packed fp32x2 instructions
          float a0, a1;
          fma2(a0, a1, __uint_as_float(x[2 * e]), __uint_as_float(x[2 * e + 1]), c, c, nm, nm);
          const float p0 = ex2_approx(a0), p1 = ex2_approx(a1);
          if ((e & 1) == 0) {
            add2(ls[0], ls[1], ls[0], ls[1], p0, p1);
          } else {
            add2(ls[2], ls[3], ls[2], ls[3], p0, p1);
          }
          x[e] = pack_bf16x2(p0, p1);
          if (e == 31) {  // keys 0-63 done: their P goes to TMEM while the rest is computed
            uint32_t (&ph)[32] = *reinterpret_cast<uint32_t(*)[32]>(&x[0]);
            tmem_st32(tS, ph);
          }
          if (e == 47) {
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(bar(B_PH0 + k));
            ATTN_TRACE(tr && it == 0, 1024 * k + 512 + 8 * j + 4);
          }
        }
        l += (ls[0] + ls[1]) + (ls[2] + ls[3]);
        ATTN_TRACE(tr && it == 0, 1024 * k + 512 + 8 * j + 3);
        {
          uint32_t (&p1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&x[32]);
          tmem_st32(tS + 32u, p1);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(bar(B_PF0 + k));
        ATTN_TRACE(tr && it == 0, 1024 * k + 512 + 8 * j + 1);
      }
      ATTN_TRACE(tr, 1024 * k + 16 * it + 2);
      if (split && k == 1) {
        // warpgroup 1's row state (reference max, sum) for warpgroup 0's merge,
        // in the Q_1 tile's space (unused with one query tile); its O stays in
        // TMEM.  Warpgroup 0 reads them after the barrier and releases O_1.
        float* ml = reinterpret_cast<float*>(gbase + kA_Q1);
        ml[row] = m_ref;
        ml[128 + row] = l;
        named_bar_arrive(3, 256);
        continue;
      }
      // Split: warpgroup 1's S products read Q_0 too; its arrival (after it
      // has waited for every one of them) lets warpgroup 0 overwrite Q_0.
      if (split) named_bar_sync(3, 256);
      // Every Q_k K^T product of the item has completed: overwrite this row of
      // Q_k with sigma(Q_k) (bf16) for the memory read, and form the fp32
      // denominator sigma(q) . z_{s-1} from the unrounded sigma.  (The z copy
      // is free again here: the warpgroup's last reads of it, in the previous
      // item, precede its O-free arrival, which precedes this item's S.)
      float den = 0.f;
      {
        float* zk = zs + 128 * k;
        zk[row] = zrow;
        named_bar_sync(1 + k, 128);
        ATTN_TRACE(tr, 1024 * k + 16 * it + 9);
        const uint32_t q = sQ(k);
        float dp[4] = {0.f, 0.f, 0.f, 0.f};
        // With position embeddings the Q tile holds rotated rows: sigma(Q) is
        // formed from the un-rotated row in global memory instead (a row past
        // the segment's end reads zeros; it is never stored).
        const int grow = (w.tq0 + k) * kTile + row;
        const uint4* gq = a.qm == nullptr || grow >= w.n_s
                              ? nullptr
                              : reinterpret_cast<const uint4*>(a.qm + w.b * a.qms[0] + w.h * a.qms[1] +
                                                               (w.seg0 + grow) * a.qms[2]);
        // Two batches of 8 chunks: the loads of a batch are in flight
        // together and its 64 elements are independent, while the code stays
        // small enough for the instruction cache (this runs once per item).
#pragma unroll 1
        for (int c8 = 0; c8 < 16; c8 += 8) {
          uint4 v[8];
          if (a.qm == nullptr) {
#pragma unroll
            for (int i = 0; i < 8; ++i) v[i] = lds128(q + swz_chunk(row, c8 + i));
          } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) v[i] = gq ? __ldg(gq + c8 + i) : make_uint4(0u, 0u, 0u, 0u);
          }
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float4 za = *reinterpret_cast<const float4*>(zk + 8 * (c8 + i));
            const float4 zb = *reinterpret_cast<const float4*>(zk + 8 * (c8 + i) + 4);
            const float zz[8] = {za.x, za.y, za.z, za.w, zb.x, zb.y, zb.z, zb.w};
            uint32_t* wp = reinterpret_cast<uint32_t*>(&v[i]);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float s0 = elu1(bf16_lo(wp[e])), s1 = elu1(bf16_hi(wp[e]));
              dp[e] = fmaf(s0, zz[2 * e], dp[e]);
              dp[e] = fmaf(s1, zz[2 * e + 1], dp[e]);
              wp[e] = pack_bf16x2(s0, s1);
            }
          }
#pragma unroll
          for (int i = 0; i < 8; ++i) sts128(q + swz_chunk(row, c8 + i), v[i]);
        }
        ATTN_TRACE(tr, 1024 * k + 16 * it + 10);
        den = (dp[0] + dp[1]) + (dp[2] + dp[3]);
        fence_proxy_async_smem();
        mbar_arrive(bar(B_SQ0 + k));
      }
      ATTN_TRACE(tr, 1024 * k + 16 * it + 3);
      // ---------------------------------------------------------------- epilogue
      mbar_wait(bar(B_MEM0 + k), (uint32_t)(it & 1));  // also implies the last P V of tile k
      ATTN_TRACE(tr, 1024 * k + 16 * it + 4);
      tc_fence_after();
      if (split) {
        // Merge the two warpgroups' softmax states: reference maxima m0, m1
        // (log2 units), sums l0, l1, unnormalised O_0, O_1 (TMEM; B_MEM0
        // complete implies warpgroup 1's products complete):
        // O = 2^(m0-m) O_0 + 2^(m1-m) O_1, l = 2^(m0-m) l0 + 2^(m1-m) l1.
        // (warpgroup 1 stored m1, l1 before the barrier above.)
        const float* ml = reinterpret_cast<const float*>(gbase + kA_Q1);
        const float m1 = ml[row], l1 = ml[128 + row];
        const bool has0 = w.nk0 > 0;  // warpgroup 0 had key tiles (O_0 written)
        const float mx = has0 ? fmaxf(m_ref, m1) : m1;
        const float a0 = has0 ? ex2_approx(m_ref - mx) : 0.f, a1 = ex2_approx(m1 - mx);
        const float lt = a0 * l + a1 * l1;
        const float gw = 1.f / (1.f + __expf(-a.beta[w.h]));
        const float wdot = (1.f - gw) / lt;
        const float wmem = den != 0.f ? gw / den : 0.f;
        const int qrow = w.tq0 * kTile + row;
        const bool valid = qrow < w.n_s;
        uint4* dst = reinterpret_cast<uint4*>(a.out + w.b * a.os[0] + w.h * a.os[1] + (w.seg0 + qrow) * a.os[2]);
        const uint32_t tO1 = tmem + lrow + 384u;
#pragma unroll 1
        for (int c8 = 0; c8 < 8; ++c8) {  // 16 columns at a time
          uint32_t r0[16], r1[16], rm[16];
          if (has0) tmem_ld16(tO + 16u * c8, r0);
          tmem_ld16(tO1 + 16u * c8, r1);
          tmem_ld16(tS + 16u * c8, rm);
          tmem_ld_wait();
          float o[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            o[e] = has0 ? fmaf(a0, __uint_as_float(r0[e]), a1 * __uint_as_float(r1[e])) : a1 * __uint_as_float(r1[e]);
          uint32_t pk[8];
#pragma unroll
          for (int e = 0; e < 8; ++e)
            pk[e] = pack_bf16x2(wmem * __uint_as_float(rm[2 * e]) + wdot * o[2 * e],
                                wmem * __uint_as_float(rm[2 * e + 1]) + wdot * o[2 * e + 1]);
          if (valid) {
            dst[2 * c8] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            dst[2 * c8 + 1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
          }
          if (a.adot != nullptr && valid) {
            const float inv_l = 1.f / lt;
            float4* ad = reinterpret_cast<float4*>(a.adot + (((long long)w.b * a.H + w.h) * a.L + w.seg0 + qrow) * 128);
#pragma unroll
            for (int e = 0; e < 4; ++e)
              ad[4 * c8 + e] = make_float4(o[4 * e] * inv_l, o[4 * e + 1] * inv_l, o[4 * e + 2] * inv_l, o[4 * e + 3] * inv_l);
          }
        }
        if (a.lse2 != nullptr && valid) a.lse2[((long long)w.b * a.H + w.h) * a.L + w.seg0 + qrow] = mx + __log2f(lt);
        // S_0, O_0 and O_1 are read out: the next item's products may overwrite them
        tc_fence_before();
        mbar_arrive(bar(B_OF0));
        mbar_arrive(bar(B_OF0 + 1));
        continue;
      }
      const float gw = 1.f / (1.f + __expf(-a.beta[w.h]));
      const float wdot = (1.f - gw) / l;
      const float wmem = den != 0.f ? gw / den : 0.f;
      const int qrow = (w.tq0 + k) * kTile + row;
      const bool valid = qrow < w.n_s;
      uint4* dst = reinterpret_cast<uint4*>(a.out + w.b * a.os[0] + w.h * a.os[1] + (w.seg0 + qrow) * a.os[2]);
      // two halves of 64 columns: four TMEM loads in flight per wait
#pragma unroll 1
      for (int c2 = 0; c2 < 4; c2 += 2) {
        uint32_t ro[64], rm[64];
        {
          uint32_t (&ro0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&ro[0]);
          uint32_t (&ro1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&ro[32]);
          uint32_t (&rm0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&rm[0]);
          uint32_t (&rm1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&rm[32]);
          tmem_ld32(tO + 32u * c2, ro0);
          tmem_ld32(tO + 32u * (c2 + 1), ro1);
          tmem_ld32(tS + 32u * c2, rm0);
          tmem_ld32(tS + 32u * (c2 + 1), rm1);
          tmem_ld_wait();
        }
        uint32_t pk[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const float v0 = wmem * __uint_as_float(rm[2 * e]) + wdot * __uint_as_float(ro[2 * e]);
          const float v1 = wmem * __uint_as_float(rm[2 * e + 1]) + wdot * __uint_as_float(ro[2 * e + 1]);
          pk[e] = pack_bf16x2(v0, v1);
        }
        if (valid) {
#pragma unroll
          for (int e = 0; e < 8; ++e) dst[4 * c2 + e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
        }
        if (a.adot != nullptr && valid) {
          const float inv_l = 1.f / l;
          float4* ad = reinterpret_cast<float4*>(a.adot + (((long long)w.b * a.H + w.h) * a.L + w.seg0 + qrow) * 128);
#pragma unroll
          for (int e = 0; e < 16; ++e)
            ad[16 * (c2 / 2) + e] =
                make_float4(__uint_as_float(ro[4 * e]) * inv_l, __uint_as_float(ro[4 * e + 1]) * inv_l,
                            __uint_as_float(ro[4 * e + 2]) * inv_l, __uint_as_float(ro[4 * e + 3]) * inv_l);
        }
      }
      if (a.lse2 != nullptr && valid) a.lse2[((long long)w.b * a.H + w.h) * a.L + w.seg0 + qrow] = m_ref + __log2f(l);
      // S_k and O_k are read out: the next item's products may overwrite them
      tc_fence_before();
      mbar_arrive(bar(B_OF0 + k));
      ATTN_TRACE(tr, 1024 * k + 16 * it + 5);
      ATTN_TRACE(tr, 1024 * k + 16 * it + 6);
    }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace tc
}  // namespace infini
