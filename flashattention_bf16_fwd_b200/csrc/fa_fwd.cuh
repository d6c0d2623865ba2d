// fa_fwd.cuh - forward pass: tiled attention with an online safe softmax, the
// repeated-max fix, a BF16 rounding point for P_bar, and the log-sum-exp.
//
// Method: "Is Flash Attention Stable?" (chibakuma.com) describes the tiling:
// Q/K/V are cut into blocks held on chip, each block is scaled and folded into
// a running result, so the N x N score matrix never reaches HBM.  "Why
// Low-Precision Transformer Training Fails" (admirer.cn summary, mechanism 2)
// places the bias in the unnormalised output P_bar V and gives the fix: when
// the row maximum of S occurs more than once, raise the shift m so every
// exponent, the maxima included, is strictly below 1.
//
// Persistent CTAs (one per SM) loop over work items; one item = one
// (batch, head) and two 128-row query tiles, processed by two softmax
// warpgroups so the tensor core works on one tile while the other tile's
// softmax runs on the CUDA cores.  An item's epilogue overlaps the next item's
// first MMAs:
//   warps 0-3  softmax warpgroup 0 (thread r owns row r: TMEM lane r)
//   warps 4-7  softmax warpgroup 1
//   warp  8    TMA producer: an item's Q tiles, then a ring of K/V stages
//   warp  9    TMEM allocator + tcgen05.mma issuer (the whole warp runs the
//              issuing loop, one elected lane executes each MMA); at d = 64
//              it issues warpgroup 0's MMAs only
//   warp 10    d = 64: tcgen05.mma issuer of warpgroup 1 (idle at d = 128)
//   warp 11    idle (it completes the third warpgroup)
// d = 64 stores O through a 128-byte-swizzled staging tile per warpgroup: each
// warp writes its 32 rows there and issues one TMA store box, so the softmax
// warps move on to the next item instead of issuing row-wise global stores.
// d = 64 runs the two warpgroups' MMA chains independently, each with its own
// issuer and its own walk over the items, and keeps two Q buffers: under a
// causal mask the second query tile of an item sees one key tile more than the
// first, so the warpgroup that takes it alternates from one item to the next
// (odd rounds swap the tiles), and the warpgroup with the shorter tile starts
// the next item instead of waiting.  d = 128 has room for neither and keeps
// one issuer that alternates the warpgroups tile by tile.
// Registers: launched at 168 per thread (384 threads); the third warpgroup
// gives back down to 104 and the two softmax warpgroups take 200 each:
// 128 * (200 + 200 + 104) = 384 * 168.
// TMEM (512 columns): S0 [0,128), S1 [128,256), O0 [256,256+d), O1 after.
// P_bar (bf16 or fp16, two per 32-bit column) overwrites the first 64 columns of S_t
// and is the A operand of O_t += P_bar V (V is the MN-major B operand).
#pragma once

#include <type_traits>

#include "sm100.cuh"

namespace fa {

struct FwdParams {
  void* o;              // [BH, N, D] of the element type
  float* lse;           // [BH, N]
  int32_t* ties;        // [BH, N] or nullptr: the detector record
  int32_t* one_hit;     // [BH, N] or nullptr: entries with P_bar == 1.0 under the final shift
  float* o_f32;         // [BH, N, D] or nullptr: O before its rounding to the element format
  int* dev_error;       // library error flag
  int BH, N, n_pairs, causal;   // BH = batch * query heads
  int H, group;         // query heads per batch entry; query heads per K/V head (1 = no sharing)
  float scale_log2;     // scale * log2(e): S -> base-2 exponent domain
  float delta_log2;     // shift added to m on repeated-max rows (0 = fix off)
  float fix_factor;     // 2^-delta_log2: P at a repeated maximum (1 - 2^-8 or, in fp16, 1 - 2^-11; 0.5; exp(-1/16))
  int fix;              // raise the shift on repeated-max rows
  int self_norm;        // divide O by the sum of the rounded P_bar instead of the unrounded P
  int near;             // detect near ties (P rounds to 1.0 in the element format) instead of exact ties of S
};

template <int D>
struct FwdLayout {
  static constexpr int kStages = (D == 64) ? 4 : 2;   // K/V ring depth
  static constexpr int kSub = D / 64;                 // 64-column sub-tiles per 128-row tile
  static constexpr int kSubBytes = 128 * 64 * 2;      // one TMA box, 16 KB
  static constexpr int kTileBytes = kSub * kSubBytes; // a 128 x D bf16 tile
  static constexpr int kQBufs = (D == 64) ? 2 : 1;    // Q buffers (d = 64: the next item's Q loads early)
  static constexpr int kQOff = 0;                     // buffer b: the tiles of warpgroups 0 and 1
  static constexpr int kKVOff = kQBufs * 2 * kTileBytes;   // stage s: K, then V
  // d = 64: O leaves through a swizzled staging tile per warpgroup (TMA store
  // of one 32-row box per warp)
  static constexpr int kOOff = kKVOff + kStages * 2 * kTileBytes;
  static constexpr int kOStage = (D == 64) ? 2 * kTileBytes : 0;
  static constexpr int kBarOff = kOOff + kOStage;
  static constexpr int kBytes = kBarOff + 256;
  static constexpr int kAlloc = kBytes + 1024;        // room to align the base to 1 KB
  static constexpr uint32_t kTmemCols = 512;
  // TMEM columns.  d = 64: S0, S1, P_bar0, P_bar1, O0, O1 each have their own,
  // so S of the next key tile can be computed as soon as the softmax has read
  // S of this one.  d = 128: O0, O1 take 256 columns and P_bar overwrites the
  // first half of S; the next S then waits for P_bar V.
  static constexpr bool kSepP = (D == 64);
  __host__ __device__ static constexpr uint32_t tm_s(int t) { return 128 * t; }
  __host__ __device__ static constexpr uint32_t tm_p(int t) { return kSepP ? 256 + 64 * t : 128 * t; }
  __host__ __device__ static constexpr uint32_t tm_o(int t) { return kSepP ? 384 + 64 * t : 256 + D * t; }
  static constexpr int kThreads = 384;
  static constexpr int kLaunchRegs = 168;       // per thread, fixed by __launch_bounds__(384, 1)
  // the producer/MMA warpgroup spills below 104 (d = 128: longer MMA
  // sequences; d = 64: two issuers)
  static constexpr uint32_t kSoftmaxRegs = 200;
  static constexpr uint32_t kOtherRegs = 104;
  static_assert(128 * (2 * kSoftmaxRegs + kOtherRegs) <= kThreads * kLaunchRegs, "register split exceeds the pool");
};

// One work item = one (batch*head, pair of query tiles).  Items are numbered
// heavy first (causal: the last query tiles see the most keys); the CTAs are
// persistent and sweep the sorted items with snake_item().  (Grouping the
// items by heads so that fewer heads' K/V stream through the L2 at once was
// measured slower: the balance of the heavy-first order matters more.)
struct FwdItem {
  int bh, q0_row, n0, n1, nmax;
};

__device__ __forceinline__ FwdItem fwd_item(const FwdParams& p, int item) {
  FwdItem it;
  const int pair = p.causal ? (p.n_pairs - 1 - item / p.BH) : item / p.BH;
  it.bh = item % p.BH;
  it.q0_row = pair * 256;
  const int n_kv = (p.N + 127) / 128;
  it.n0 = p.causal ? min(2 * pair + 1, n_kv) : n_kv;
  it.n1 = (it.q0_row + 128 < p.N) ? (p.causal ? min(2 * pair + 2, n_kv) : n_kv) : 0;
  it.nmax = max(it.n0, it.n1);
  return it;
}

// The query tile (0 or 1 of the item) that softmax warpgroup t takes in round
// rnd of the CTA's item walk.  d = 64 swaps them in odd rounds, so that the
// longer causal tile alternates between the warpgroups.
template <int D>
__device__ __forceinline__ int fwd_tile_of(int t, int rnd) {
  return FwdLayout<D>::kSepP ? (t ^ (rnd & 1)) : t;
}

// The smallest value below 1 that rounds to 1.0 in E's format (ties to even):
// 1 - 2^-9 in bf16, 1 - 2^-12 in fp16.  P at or above it gives P_bar == 1.
template <typename E>
__device__ __forceinline__ constexpr float rounds_to_one() {
  return E::kMmaFmt == 1 ? 0.998046875f : 0.999755859375f;
}

// E: the element format (ElemBF16 or ElemF16) of Q, K, V, O and of P_bar.
// kVariants: compiled with the code of fix_mode 4 (self-normalised) and 5
// (near ties) and with the debug records (tie record, P_bar == 1 count, O
// before rounding); the other instantiation, used for fix_mode 0-3 without
// records, leaves all of it out.
template <int D, bool kVariants, typename E = ElemBF16>
__global__ void __launch_bounds__(384, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                  const FwdParams p) {
  using L = FwdLayout<D>;
  const float kNegInf = -__int_as_float(0x7f800000);
  constexpr float kLn2 = 0.69314718055994531f;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* q_full = bars;         // [kQBufs]
  uint64_t* q_empty = bars + 2;    // [kQBufs]
  uint64_t* kv_full = bars + 4;
  uint64_t* kv_empty = kv_full + L::kStages;
  uint64_t* s_full = kv_empty + L::kStages;  // [2]
  uint64_t* p_full = s_full + 2;             // [2]
  uint64_t* o_done = p_full + 2;             // [2]
  uint64_t* o_free = o_done + 2;             // [2]
  uint64_t* s_free = o_free + 2;             // [2] the softmax has read S_t (d = 64)
  uint64_t* mma_done = s_free + 2;          // [2] one per MMA issuer
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int n_items = p.n_pairs * p.BH;
  const int warp = int(warp_id());
  const int lane = int(lane_id());

  if (threadIdx.x == 0) {
    for (int b = 0; b < L::kQBufs; ++b) {
      mbar_init(&q_full[b], 1);
      mbar_init(&q_empty[b], L::kSepP ? 2 : 1);   // d = 64: both MMA issuers
    }
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], L::kSepP ? 2 : 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&s_full[t], 1);
      mbar_init(&p_full[t], 128);
      mbar_init(&o_done[t], 1);
      mbar_init(&o_free[t], 128);
      mbar_init(&s_free[t], 128);
    }
    mbar_init(&mma_done[0], 1);
    mbar_init(&mma_done[1], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(tmem_slot, L::kTmemCols);
    tmem_relinquish();
  }
  if (warp == 8 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // set-up above touched no global memory; from here on the previous
  // kernel's writes are needed
  grid_dep_wait();
  grid_dep_launch();
  const Watchdog wd{abort_flag, p.dev_error};

  if (warp >= 8) {
    // Producer and MMA warps need few registers; give them back first.
    regs_set<L::kOtherRegs, L::kLaunchRegs>();
    if (warp == 8) {
      // ------------------------------------------------------------- producer
      if (lane == 0) {
        const uint64_t pol_q = l2_policy_evict_first();
        const uint64_t pol_kv = l2_policy_evict_last();
        uint32_t kv_cnt = 0;   // K/V tiles loaded so far by this CTA
        uint32_t n_done = 0;   // items started
        bool ok = true;
        for (int rnd = 0, item = snake_item(0); ok && item < n_items; item = snake_item(++rnd), ++n_done) {
          const FwdItem w = fwd_item(p, item);
          // grouped-query layout: query head h reads K/V head h / group
          const int kv_bh = (w.bh / p.H) * (p.H / p.group) + (w.bh % p.H) / p.group;
          // the S MMAs of the item kQBufs back must be done with this Q buffer
          const uint32_t qb = n_done % L::kQBufs;
          if (!(ok = mbar_wait(&q_empty[qb], ((n_done / L::kQBufs) & 1) ^ 1, wd))) break;
          const int nq = (w.n1 > 0) ? 2 : 1;
          mbar_arrive_expect_tx(&q_full[qb], uint32_t(nq * L::kTileBytes));
          for (int qt = 0; qt < nq; ++qt)   // query tile qt into the buffer of the warpgroup that takes it
            for (int s = 0; s < L::kSub; ++s)
              tma_load_3d(smem + L::kQOff + (qb * 2 + fwd_tile_of<D>(qt, rnd)) * L::kTileBytes + s * L::kSubBytes,
                          &tm_q, &q_full[qb], s * 64, w.q0_row + qt * 128, w.bh, pol_q);
          for (int j = 0; j < w.nmax; ++j, ++kv_cnt) {
            const uint32_t st = kv_cnt % L::kStages;
            if (!(ok = mbar_wait(&kv_empty[st], ((kv_cnt / L::kStages) & 1) ^ 1, wd))) break;
            mbar_arrive_expect_tx(&kv_full[st], uint32_t(2 * L::kTileBytes));
            uint8_t* sk = smem + L::kKVOff + st * 2 * L::kTileBytes;
            uint8_t* sv = sk + L::kTileBytes;
            for (int s = 0; s < L::kSub; ++s) {
              tma_load_3d(sk + s * L::kSubBytes, &tm_k, &kv_full[st], s * 64, j * 128, kv_bh, pol_kv);
              tma_load_3d(sv + s * L::kSubBytes, &tm_v, &kv_full[st], s * 64, j * 128, kv_bh, pol_kv);
            }
          }
        }
      }
    } else if (L::kSepP && (warp == 9 || warp == 10)) {
      // ------------------------------------------ d = 64: MMA issuers, one per
      // softmax warpgroup, each walking the items on its own.  Q buffers and
      // K/V stages are released once both issuers are done with them (their
      // empty barriers count two arrivals); a warpgroup whose tile of an item
      // is shorter goes on to the next item while the other finishes.
      {
        // The whole warp runs the loop (warp-uniform operands and waits); one
        // elected lane executes each MMA.  From lane 0 alone, a tile's eight
        // P_bar V MMAs took 600-1100 cycles to issue, which delayed the end
        // of every item.
        auto wait = [&](uint64_t* bar, uint32_t parity) {
          return __all_sync(0xffffffffu, mbar_wait(bar, parity, wd));
        };
        const int t = warp - 9;
        constexpr uint32_t kIdS = make_idesc(128, 128, 0, 0, E::kMmaFmt);
        constexpr uint32_t kIdPV = make_idesc(128, D, 0, 1, E::kMmaFmt);
        const uint64_t dq0 = make_sdesc_sw128(smem_u32(smem + L::kQOff), 16, 1024);
        const uint64_t dk0 = make_sdesc_sw128(smem_u32(smem + L::kKVOff), 16, 1024);
        const uint64_t dv0 = make_sdesc_sw128(smem_u32(smem + L::kKVOff + L::kTileBytes), L::kSubBytes, 1024);
        uint32_t qb = 0;
        auto issue_s = [&](uint32_t st) {
          const uint64_t a = sdesc_add(dq0, (qb * 2 + t) * L::kTileBytes);
          const uint64_t b = sdesc_add(dk0, st * 2 * L::kTileBytes);
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const uint32_t off = (k >> 2) * L::kSubBytes + (k & 3) * 32;
            umma_ss_warp(tmem + L::tm_s(t), sdesc_add(a, off), sdesc_add(b, off), kIdS, k > 0);
          }
          umma_commit_warp(&s_full[t]);
        };
        auto issue_pv = [&](uint32_t st, int j) {
          const uint64_t b = sdesc_add(dv0, st * 2 * L::kTileBytes);
#pragma unroll
          for (int k = 0; k < 8; ++k)
            umma_ts_warp(tmem + L::tm_o(t), tmem + L::tm_p(t) + k * 8, sdesc_add(b, k * 2048), kIdPV,
                         (j > 0 || k > 0) ? 1u : 0u);
          umma_commit_warp(&o_done[t]);
        };
        uint32_t kv_cnt = 0, it_cnt = 0, ep_cnt = 0, n_done = 0;
        bool ok = true;
        for (int rnd = 0, item = snake_item(0); ok && item < n_items; item = snake_item(++rnd), ++n_done) {
          const FwdItem w = fwd_item(p, item);
          const int nt = fwd_tile_of<D>(t, rnd) ? w.n1 : w.n0;   // key tiles of this warpgroup's query tile
          qb = n_done % L::kQBufs;
          if (!(ok = wait(&q_full[qb], (n_done / L::kQBufs) & 1))) break;
          if (nt > 0) {
            if (!(ok = wait(&kv_full[kv_cnt % L::kStages], (kv_cnt / L::kStages) & 1))) break;
            if (it_cnt > 0 && !(ok = wait(&s_free[t], (it_cnt - 1) & 1))) break;
            tc_fence_after();
            issue_s(kv_cnt % L::kStages);
          }
          if (nt <= 1) umma_commit_warp(&q_empty[qb]);     // this issuer's S MMAs of the item are issued
          for (int j = 0; ok && j < w.nmax; ++j) {
            const uint32_t st = (kv_cnt + j) % L::kStages;
            if (j + 1 < nt) {
              const uint32_t nxt = kv_cnt + j + 1;
              if (!(ok = wait(&kv_full[nxt % L::kStages], (nxt / L::kStages) & 1) &&
                         wait(&s_free[t], (it_cnt + j) & 1)))
                break;
              tc_fence_after();
              issue_s(nxt % L::kStages);
              if (j + 2 == nt) umma_commit_warp(&q_empty[qb]);
            }
            if (j < nt) {
              if (!(ok = wait(&p_full[t], (it_cnt + j) & 1))) break;
              if (j == 0 && !(ok = wait(&o_free[t], (ep_cnt & 1) ^ 1))) break;
              tc_fence_after();
              issue_pv(st, j);
            }
            // a key tile this warpgroup does not use (its query tile sees
            // fewer): wait until it is loaded before releasing its stage, so
            // that this issuer's arrival belongs to this use of the stage and
            // it never runs a use ahead of the other issuer
            if (j >= nt && !(ok = wait(&kv_full[st], ((kv_cnt + j) / L::kStages) & 1))) break;
            umma_commit_warp(&kv_empty[st]);     // this issuer is done with the stage
          }
          kv_cnt += w.nmax;
          it_cnt += nt;
          ep_cnt += (nt > 0) ? 1 : 0;
        }
        umma_commit_warp(&mma_done[t]);
        wait(&mma_done[t], 0);
      }
      __syncwarp();
    } else if (!L::kSepP && warp == 9) {
      // ------------------------------------------------- d = 128: MMA issuer
      // Per key tile j: P_bar_0 V, S_0 of tile j+1 (it overwrites P_bar_0),
      // P_bar_1 V, S_1 of tile j+1; the two warpgroups alternate at the
      // tensor core.
      {
        // the whole warp runs the loop; one elected lane executes each MMA
        auto wait = [&](uint64_t* bar, uint32_t parity) {
          return __all_sync(0xffffffffu, mbar_wait(bar, parity, wd));
        };
        constexpr uint32_t kIdS = make_idesc(128, 128, 0, 0, E::kMmaFmt);   // Q K^T: both K-major
        constexpr uint32_t kIdPV = make_idesc(128, D, 0, 1, E::kMmaFmt);    // P_bar V: V is MN-major
        // Descriptors are built once; each MMA only advances the start address.
        const uint64_t dq0 = make_sdesc_sw128(smem_u32(smem + L::kQOff), 16, 1024);
        const uint64_t dk0 = make_sdesc_sw128(smem_u32(smem + L::kKVOff), 16, 1024);
        const uint64_t dv0 = make_sdesc_sw128(smem_u32(smem + L::kKVOff + L::kTileBytes), L::kSubBytes, 1024);
        auto issue_s = [&](int t, uint32_t st) {
          const uint64_t a = sdesc_add(dq0, t * L::kTileBytes);
          const uint64_t b = sdesc_add(dk0, st * 2 * L::kTileBytes);
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const uint32_t off = (k >> 2) * L::kSubBytes + (k & 3) * 32;
            umma_ss_warp(tmem + L::tm_s(t), sdesc_add(a, off), sdesc_add(b, off), kIdS, k > 0);
          }
          umma_commit_warp(&s_full[t]);
        };
        auto issue_pv = [&](int t, uint32_t st, int j) {
          const uint64_t b = sdesc_add(dv0, st * 2 * L::kTileBytes);
#pragma unroll
          for (int k = 0; k < 8; ++k)
            umma_ts_warp(tmem + L::tm_o(t), tmem + L::tm_p(t) + k * 8, sdesc_add(b, k * 2048), kIdPV,
                         (j > 0 || k > 0) ? 1u : 0u);
          umma_commit_warp(&o_done[t]);
        };
        uint32_t kv_cnt = 0;           // K/V tiles consumed
        uint32_t it_cnt[2] = {0, 0};   // softmax iterations per query tile
        uint32_t ep_cnt[2] = {0, 0};   // items finished per query tile (epilogues)
        uint32_t n_done = 0;
        bool ok = true;
        for (int rnd = 0, item = snake_item(0); ok && item < n_items; item = snake_item(++rnd), ++n_done) {
          const FwdItem w = fwd_item(p, item);
          const int nt[2] = {w.n0, w.n1};
          if (!(ok = wait(q_full, n_done & 1) &&
                     wait(&kv_full[kv_cnt % L::kStages], (kv_cnt / L::kStages) & 1)))
            break;
          tc_fence_after();
          for (int t = 0; t < 2; ++t)
            if (nt[t] > 0) issue_s(t, kv_cnt % L::kStages);
          if (w.nmax == 1) umma_commit_warp(q_empty);
          for (int j = 0; ok && j < w.nmax; ++j) {
            const uint32_t st = (kv_cnt + j) % L::kStages;
            const uint32_t stn = (kv_cnt + j + 1) % L::kStages;
            for (int t = 0; t < 2; ++t) {
              if (j < nt[t]) {
                if (!(ok = wait(&p_full[t], (it_cnt[t] + j) & 1))) break;
                // the first P_bar V of an item overwrites O_t: the previous
                // item's epilogue must have read it
                if (j == 0 && !(ok = wait(&o_free[t], (ep_cnt[t] & 1) ^ 1))) break;
                tc_fence_after();
                issue_pv(t, st, j);
              }
              if (t == 0 && j + 1 < w.nmax) {
                const uint32_t nxt = kv_cnt + j + 1;
                if (!(ok = wait(&kv_full[stn], (nxt / L::kStages) & 1))) break;
                tc_fence_after();
                if (j + 1 < nt[0]) issue_s(0, stn);   // S_0 of tile j+1 overwrites P_bar_0 after P_bar V
              }
              if (t == 1) {
                umma_commit_warp(&kv_empty[st]);
                if (j + 1 < nt[1]) issue_s(1, stn);
                if (j + 2 == w.nmax) umma_commit_warp(q_empty);   // the item's last S MMAs are issued
              }
            }
          }
          kv_cnt += w.nmax;
          for (int t = 0; t < 2; ++t) {
            it_cnt[t] += nt[t];
            ep_cnt[t] += (nt[t] > 0) ? 1 : 0;
          }
        }
        // Every MMA must be finished before TMEM is released.
        umma_commit_warp(&mma_done[0]);
        wait(&mma_done[0], 0);
      }
      __syncwarp();
    }
  } else {
    regs_set<L::kSoftmaxRegs, L::kLaunchRegs>();
    // --------------------------------------------------- softmax warpgroups
    const int t = warp >> 2;
    const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
    const uint32_t t_s = tmem + lane_base + L::tm_s(t);
    const uint32_t t_p = tmem + lane_base + L::tm_p(t);
    const uint32_t t_o = tmem + lane_base + L::tm_o(t);
    const float sl2 = p.scale_log2;
    // 2^-delta: on a row whose maximum becomes repeated in the current tile,
    // P is computed with the plain shift and then multiplied by this, which is
    // the same as raising m by delta (rows repeated before the tile take the
    // raised shift in the exponent instead); each maximum lands on this value
    // (1 - 2^-8 for fix_mode 1 in bf16, 1 - 2^-11 in fp16).
    const float kFixFactor = p.fix_factor;
    uint32_t it_cnt = 0;   // softmax iterations done by this warpgroup
    bool ok = true;

    for (int rnd = 0, item = snake_item(0); ok && item < n_items; item = snake_item(++rnd)) {
      const FwdItem w = fwd_item(p, item);
      const int qt = fwd_tile_of<D>(t, rnd);   // which of the item's two query tiles
      const int n_t = qt ? w.n1 : w.n0;
      if (n_t == 0) continue;
      const int row = w.q0_row + qt * 128 + (warp & 3) * 32 + lane;
      const int limit = p.causal ? min(row, p.N - 1) : p.N - 1;   // last visible key

      float m = kNegInf;    // running max of the raw scores S
      int cnt = 0;          // how many seen scores equal m
      float ms = kNegInf;   // m * scale_log2: the shift without the fix
      bool raised = false;  // the shift in use is ms + delta (fix active on this row)
      float l = 0.f;        // running sum of the unrounded P, relative to the shift in use
      bool ever_repeated = false;   // the running max occurred >= 2 times at some tile
      float l_bar = 0.f;    // running sum of the rounded P_bar (self-normalised mode only)
      int cnt_near = 0;     // near-tie mode: 2 when two or more entries so far have P rounding to 1 under the plain shift
      float s2 = kNegInf;   // near-tie mode: second largest raw score so far (a repeated maximum counts twice)
      int hits = 0;         // entries packed as P_bar == 1.0 since the shift last moved (one_hit record)

      for (int j = 0; j < n_t; ++j) {
        const uint32_t ph = (it_cnt + j) & 1;
        ok = __all_sync(0xffffffffu, mbar_wait(&s_full[t], ph, wd));
        if (!ok) break;
        tc_fence_after();
        uint32_t r[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(t_s + c * 32, r[c]);
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld_wait(r[c]);
        if (L::kSepP) {                                // S_t is in registers: the next S may overwrite it
          tc_fence_before();
          mbar_arrive(&s_free[t]);
        }
        float s[128];
#pragma unroll
        for (int i = 0; i < 128; ++i) s[i] = __uint_as_float(r[i >> 5][i & 31]);

        const int key0 = j * 128;
        const bool masked = key0 + 127 > limit;
        if (masked) {
#pragma unroll
          for (int i = 0; i < 128; ++i) s[i] = (key0 + i > limit) ? kNegInf : s[i];
        }
        // tile maximum: eight 16-wide 3-input max chains, then a short tree
        float mx[8];
#pragma unroll
        for (int g = 0; g < 8; ++g) {
          float a = fmax3(s[16 * g], s[16 * g + 1], s[16 * g + 2]);
#pragma unroll
          for (int i = 3; i < 15; i += 2) a = fmax3(a, s[16 * g + i], s[16 * g + i + 1]);
          mx[g] = fmaxf(a, s[16 * g + 15]);
        }
        const float mt = fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7]));
        const float m_new = fmaxf(m, mt);
        const float ms_new = (m_new == kNegInf) ? 0.f : m_new * sl2;
        // near-tie mode: the largest score of the tile below its maximum
        float s2x = kNegInf;
        if (kVariants && p.near) {
#pragma unroll
          for (int i = 0; i < 128; ++i) s2x = fmaxf(s2x, (s[i] < mt) ? s[i] : kNegInf);
        }

        // A row whose running maximum is already repeated and does not move in
        // this tile keeps the raised shift whatever the tile holds, so its P
        // is computed with the raised shift directly (the exponent minus delta:
        // any maximum in this tile rounds to 2^-delta on the P_bar grid all the
        // same).
        // Only rows that become repeated in this tile need the rare path.
        const bool raise_early = p.fix && m == m_new && ((kVariants && p.near) ? cnt_near : cnt) >= 2;
        const float msh = raise_early ? ms_new + p.delta_log2 : ms_new;
        // P = 2^(S*scale_log2 - shift); the row sum and the count of entries
        // equal to the tile max ride along as independent packed adds
        uint64_t sum2[4] = {0, 0, 0, 0};
        uint64_t eq2[2] = {0, 0};
        const uint64_t sl2_2 = f2_pack(sl2, sl2);
        const uint64_t nmsh_2 = f2_pack(-msh, -msh);
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          // x = S * scale_log2 - shift: one packed FMA per pair at d = 128; at
          // d = 64 the packed form pushes the softmax past its register budget
          float x0, x1;
          if constexpr (D == 128) {
            f2_unpack(f2_fma(f2_pack(s[2 * i], s[2 * i + 1]), sl2_2, nmsh_2), x0, x1);
          } else {
            x0 = fmaf(s[2 * i], sl2, -msh);
            x1 = fmaf(s[2 * i + 1], sl2, -msh);
          }
          const float e0 = (s[2 * i] == mt) ? 1.f : 0.f;
          const float e1 = (s[2 * i + 1] == mt) ? 1.f : 0.f;
          eq2[i & 1] = f2_add(eq2[i & 1], f2_pack(e0, e1));
          s[2 * i] = ex2(x0);
          s[2 * i + 1] = ex2(x1);
          sum2[i & 3] = f2_add(sum2[i & 3], f2_pack(s[2 * i], s[2 * i + 1]));
        }
        float ea, eb;
        f2_unpack(f2_add(eq2[0], eq2[1]), ea, eb);
        const int ct = (mt == kNegInf) ? 0 : int(ea + eb);
        int c_new = (m == m_new ? cnt : 0) + (mt == m_new ? ct : 0);
        if (m_new == kNegInf) c_new = 0;
        // near-tie mode: the row has two or more entries whose P under the
        // plain shift rounds to 1.0 in the element format (P >= 1 - 2^-9 in
        // bf16, 1 - 2^-12 in fp16) exactly when its second largest score
        // does; the two largest scores are carried across key tiles, so
        // partners in earlier tiles still count after the maximum moves
        int cn_new = 0;
        float s2_new = kNegInf;
        if (kVariants && p.near) {
          const float s2t = (ct >= 2) ? mt : s2x;
          s2_new = (m > mt) ? fmaxf(s2, mt) : ((mt > m) ? fmaxf(m, s2t) : mt);
          cn_new = (s2_new != kNegInf && ex2(fmaf(s2_new, sl2, -ms_new)) >= rounds_to_one<E>()) ? 2 : 0;
        }
        const int det = (kVariants && p.near) ? cn_new : c_new;
        ever_repeated |= (det >= 2);
        const bool raise = p.fix && det >= 2;
        f2_unpack(f2_add(f2_add(sum2[0], sum2[1]), f2_add(sum2[2], sum2[3])), ea, eb);
        float rs = ea + eb;
        // Rare path: a row that became repeated in this tile had its P computed
        // with the plain shift; it is packed scaled by 2^-delta, which is the
        // raised shift (the scaled pack runs only in warps that need it)
        const bool rare = __any_sync(0xffffffffu, raise && !raise_early);
        const float pf = (raise && !raise_early) ? kFixFactor : 1.f;
        if (raise && !raise_early) rs *= kFixFactor;
        // rescale of the running O and l: exact, whenever the shift moves
        float alpha = ex2(ms - ms_new);
        if (raise != raised) alpha = raise ? alpha * kFixFactor : alpha / kFixFactor;
        l = l * alpha + rs;
        if (j > 0) {
          // P_bar V of tile j-1 must be finished: it read the P_bar buffer and
          // O_t must hold its result before O_t is rescaled
          ok = __all_sync(0xffffffffu, mbar_wait(&o_done[t], (it_cnt + j - 1) & 1, wd));
          if (!ok) break;
          tc_fence_after();
        }
        float rs_bar = 0.f;
        // one_hit record: a move of the shift rescales everything packed so
        // far by alpha != 1, so only entries packed under the final shift
        // enter O with weight P_bar; count those that are exactly 1.0
        const bool moved = (ms_new != ms) || (raise != raised);
        int th = 0;
        auto pack_store = [&](auto scaled) {
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              float a = s[c * 32 + 2 * i], b = s[c * 32 + 2 * i + 1];
              if (decltype(scaled)::value) {
                a *= pf;
                b *= pf;
              }
              pk[i] = E::pack(a, b);
            }
            if (kVariants && p.one_hit) {
#pragma unroll
              for (int i = 0; i < 16; ++i)
                th += int((pk[i] & 0xffffu) == E::kOneBits) + int((pk[i] >> 16) == E::kOneBits);
            }
            if (kVariants && p.self_norm) {
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const float2 pp = E::unpack(pk[i]);
                rs_bar += pp.x + pp.y;
              }
            }
            tmem_st16(t_p + c * 16, pk);
          }
        };
        if (rare)
          pack_store(std::true_type{});
        else
          pack_store(std::false_type{});
        l_bar = l_bar * alpha + rs_bar;
        hits = (moved ? 0 : hits) + th;
        if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
          const uint64_t a2 = f2_pack(alpha, alpha);
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld32(t_o + c * 32, o);
            tmem_ld_wait(o);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              float y0, y1;
              f2_unpack(f2_mul(f2_pack(__uint_as_float(o[2 * i]), __uint_as_float(o[2 * i + 1])), a2), y0, y1);
              o[2 * i] = __float_as_uint(y0);
              o[2 * i + 1] = __float_as_uint(y1);
            }
            tmem_st32(t_o + c * 32, o);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&p_full[t]);
        m = m_new;
        cnt = c_new;
        cnt_near = cn_new;
        s2 = s2_new;
        ms = ms_new;
        raised = raise;
      }
      if (!ok) break;

      // epilogue: O = O_acc / l -> bf16; LSE in natural-log units
      ok = __all_sync(0xffffffffu, mbar_wait(&o_done[t], (it_cnt + n_t - 1) & 1, wd));
      if (!ok) break;
      tc_fence_after();
      uint32_t ow[D / 2];
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(t_o + c * 32, o);
        tmem_ld_wait(o);
        const float inv_l = 1.f / ((kVariants && p.self_norm) ? l_bar : l);
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * inv_l);
#pragma unroll
        for (int i = 0; i < 16; ++i) ow[c * 16 + i] = E::pack(__uint_as_float(o[2 * i]), __uint_as_float(o[2 * i + 1]));
        if (kVariants && p.o_f32 && row < p.N) {   // the values whose rounding O is
          uint4* dst = reinterpret_cast<uint4*>(p.o_f32 + (size_t(w.bh) * p.N + row) * D + c * 32);
#pragma unroll
          for (int i = 0; i < 8; ++i) dst[i] = make_uint4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
        }
      }
      // O_t is in registers: the next item's first P_bar V may overwrite it
      tc_fence_before();
      mbar_arrive(&o_free[t]);
      if constexpr (L::kSepP) {
        // each warp stages its 32 rows (128-byte swizzle) and lane 0 stores
        // them with one TMA box; rows past N are clipped by the tensor map
        uint8_t* stg = smem + L::kOOff + t * L::kTileBytes + (warp & 3) * 4096;
        if (lane == 0) bulk_wait_read<0>();        // this warp's previous store has read the box
        __syncwarp();
#pragma unroll
        for (int c = 0; c < 8; ++c)
          *reinterpret_cast<uint4*>(stg + lane * 128 + ((c ^ (lane & 7)) << 4)) =
              make_uint4(ow[4 * c], ow[4 * c + 1], ow[4 * c + 2], ow[4 * c + 3]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_3d(&tm_o, stg, 0, w.q0_row + qt * 128 + (warp & 3) * 32, w.bh);
          bulk_commit();
        }
      } else if (row < p.N) {
        uint4* dst = reinterpret_cast<uint4*>(static_cast<typename E::T*>(p.o) + (size_t(w.bh) * p.N + row) * D);
#pragma unroll
        for (int i = 0; i < D / 8; ++i) dst[i] = make_uint4(ow[4 * i], ow[4 * i + 1], ow[4 * i + 2], ow[4 * i + 3]);
      }
      if (row < p.N) {
        p.lse[size_t(w.bh) * p.N + row] = (ms + (raised ? p.delta_log2 : 0.f) + lg2(l)) * kLn2;
        if (kVariants && p.ties)
          p.ties[size_t(w.bh) * p.N + row] = cnt | (raised ? (1 << 29) : 0) | (ever_repeated ? (1 << 30) : 0);
        if (kVariants && p.one_hit) p.one_hit[size_t(w.bh) * p.N + row] = hits;
      }
      it_cnt += n_t;
    }
    if (L::kSepP && lane == 0) bulk_wait<0>();     // every O store has landed
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

}  // namespace fa
