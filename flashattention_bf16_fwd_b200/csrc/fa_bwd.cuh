// fa_bwd.cuh - backward pass that recomputes P from the log-sum-exp.
//
// The yicaiai article (sections 3.4 and 4.3) names the softmax recomputation
// path and the gradients d loss/dQ, d loss/dK that flow through it.  With
// L = LSE from the forward pass, per (query i, key j):
//   P_ij = exp(scale S_ij - L_i),  dP = dO V^T,  D_i = sum_k dO_ik O_ik,
//   dS = P * (dP - D),  dV = P^T dO,  dK = scale dS^T Q,  dQ = scale dS K.
// Three kernels:
//   fa_bwd_pre_kernel  D_i and a zeroed FP32 dQ accumulator (HBM-bound)
//   fa_bwd_kernel      one CTA per (batch*head, 128-key tile); loops over the
//                      query tiles that see those keys; five tcgen05 MMAs per
//                      step; dK, dV stay in TMEM; dQ is added into the FP32
//                      accumulator with TMA reduce-add from shared memory
//   fa_bwd_dq_kernel   dQ = scale * accumulator -> bf16 (HBM-bound)
//
// fa_bwd_kernel roles and TMEM use are described above the kernel.
#pragma once

#include "sm100.cuh"

namespace fa {

// D_i = sum_k dO_ik O_ik in FP32; also zeroes the FP32 dQ accumulator.
// Eight threads per row; each covers d/8 consecutive elements.
template <typename E>
__global__ void __launch_bounds__(256) fa_bwd_pre_kernel(const typename E::T* __restrict__ o,
                                                         const typename E::T* __restrict__ dout,
                                                         float* __restrict__ dsum, float* __restrict__ dq_acc,
                                                         long long rows, int d) {
  grid_dep_wait();
  grid_dep_launch();
  const long long tid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long row = tid >> 3;
  const int sub = int(tid & 7);
  float acc = 0.f;
  if (row < rows) {
    const int per = d >> 3;   // 8 or 16 elements
    const size_t base = size_t(row) * d + size_t(sub) * per;
    for (int c = 0; c < per; c += 8) {
      const uint4 a = *reinterpret_cast<const uint4*>(o + base + c);
      const uint4 b = *reinterpret_cast<const uint4*>(dout + base + c);
      const uint32_t* a2 = reinterpret_cast<const uint32_t*>(&a);
      const uint32_t* b2 = reinterpret_cast<const uint32_t*>(&b);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 fa = E::unpack(a2[i]);
        const float2 fb = E::unpack(b2[i]);
        acc = fmaf(fa.x, fb.x, acc);
        acc = fmaf(fa.y, fb.y, acc);
      }
      float4* z = reinterpret_cast<float4*>(dq_acc + base + c);
      z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
      z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  acc += __shfl_xor_sync(0xffffffffu, acc, 1);
  acc += __shfl_xor_sync(0xffffffffu, acc, 2);
  acc += __shfl_xor_sync(0xffffffffu, acc, 4);
  if (row < rows && sub == 0) dsum[row] = acc;
}

// dQ = scale * accumulator, eight elements per thread.
template <typename E>
__global__ void __launch_bounds__(256) fa_bwd_dq_kernel(const float* __restrict__ acc,
                                                        typename E::T* __restrict__ dq, float scale,
                                                        long long n8) {
  grid_dep_wait();
  grid_dep_launch();
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n8) return;
  const float4 a = reinterpret_cast<const float4*>(acc)[2 * i];
  const float4 b = reinterpret_cast<const float4*>(acc)[2 * i + 1];
  uint4 w;
  w.x = E::pack(a.x * scale, a.y * scale);
  w.y = E::pack(a.z * scale, a.w * scale);
  w.z = E::pack(b.x * scale, b.y * scale);
  w.w = E::pack(b.z * scale, b.w * scale);
  reinterpret_cast<uint4*>(dq)[i] = w;
}

struct BwdParams {
  const float* lse;     // [BH, N] natural log
  const float* dsum;    // [BH, N] D_i
  float* dq_acc;        // [BH, N, D] FP32
  void* dk;             // [BH, N, D] of the element type
  void* dv;             // [BH, N, D] of the element type
  int* dev_error;
  int BH, N, n_kv, causal;   // BH = batch * K/V heads
  int H, group;         // query heads per batch entry; query heads per K/V head (1 = no sharing)
  float scale, scale_log2;
  int after_pre;        // 1: launched right after fa_bwd_pre_kernel on the same stream
};

template <int D>
struct BwdLayout {
  static constexpr int kSub = D / 64;
  static constexpr int kSubBytes = 128 * 64 * 2;
  static constexpr int kTileBytes = kSub * kSubBytes;
  // d=64 double-buffers K/V so the next item's keys load during this one;
  // d=128 has no room and keeps one dO buffer, refilled after dV.
  static constexpr int kKVStages = (D == 64) ? 2 : 1;
  static constexpr int kDOStages = (D == 64) ? 2 : 1;
  // Q_i (with its LSE and D rows) is loaded up to kQStages steps ahead;
  // d=64 has room for a third stage, which hides the load behind a full step.
  static constexpr int kQStages = (D == 64) ? 3 : 2;
  static constexpr int kKVOff = 0;                          // stage s: K, then V
  static constexpr int kQOff = kKVStages * 2 * kTileBytes;
  static constexpr int kDOOff = kQOff + kQStages * kTileBytes;
  static constexpr int kDSOff = kDOOff + kDOStages * kTileBytes;   // dS, [128 keys][128 queries] bf16, MN-major
  static constexpr int kStatOff = kDSOff + 2 * kSubBytes;  // kQStages x (-LSE*log2e, D) x 128 floats
  // dQ staging for the TMA reduce-add: per drain warp two 32 x 32 FP32 boxes
  static constexpr int kStageBox = 32 * 32 * 4;
  static constexpr int kDQStageOff = kStatOff + kQStages * 2 * 128 * 4;
  static constexpr int kBarOff = kDQStageOff + 4 * 2 * kStageBox;
  static constexpr int kBytes = kBarOff + 256;
  static_assert(kBytes <= 227 * 1024, "shared memory layout exceeds 227 KB");
  static constexpr int kAlloc = kBytes;                    // base is 1 KB aligned by declaration
  static constexpr uint32_t kTmemCols = 512;
  static constexpr int kThreads = 512;
  static constexpr int kLaunchRegs = 128;                  // per thread, fixed by __launch_bounds__(512, 1)
  static constexpr uint32_t kComputeRegs = 152;
  static constexpr uint32_t kDrainRegs = 112;
  static constexpr uint32_t kOtherRegs = 96;
  static_assert(128 * (2 * kComputeRegs + kDrainRegs + kOtherRegs) <= kThreads * kLaunchRegs,
                "register split exceeds the pool");
  // TMEM columns.  d = 64: P_bar^T has its own 64 columns, so S of the next
  // query tile can be computed while this tile's dS is formed.  d = 128: no
  // room; P_bar^T overwrites half of each S half and dQ reuses dP^T.
  static constexpr bool kWide = (D == 128);
  static constexpr uint32_t kTmS = 0, kTmDP = 128, kTmDV = 256, kTmDK = 256 + D;
  static constexpr uint32_t kTmDQ = kWide ? 128 : 384;
  static constexpr uint32_t kTmPT = kWide ? 0 : 448;
  // column of P_bar^T / dS^T for MMA K-step k (16 queries = 8 columns): the
  // query half h = k / 4 was written by the warps that own that half
  __host__ __device__ static constexpr uint32_t pt_col(int k) {
    return kWide ? kTmS + 64 * (k >> 2) + 8 * (k & 3) : kTmPT + 8 * k;
  }
  __host__ __device__ static constexpr uint32_t dst_col(int k) { return kTmDP + 64 * (k >> 2) + 8 * (k & 3); }
};

// One work item = one (batch*K/V head, 128-key tile).  It loops over the
// query tiles that see those keys, for each query head of the group that
// shares the K/V head (dK, dV accumulate over all of them): n_it steps.
struct BwdItem {
  int bh, kv_tile, key0, i_start, n_it_head, n_it;
};

__device__ __forceinline__ BwdItem bwd_item_at(const BwdParams& p, int bh, int kv_tile) {
  BwdItem w;
  w.bh = bh;
  w.kv_tile = kv_tile;
  w.key0 = kv_tile * 128;
  const int n_q = (p.N + 127) / 128;
  w.i_start = p.causal ? kv_tile : 0;
  w.n_it_head = n_q - w.i_start;
  w.n_it = w.n_it_head * p.group;
  return w;
}

// The sequence of work items a persistent CTA takes; every role of the CTA
// walks the same sequence.
//  - Default: items are numbered heavy first, key tile major (causal: the
//    first key tiles are seen by the most query tiles), and the CTAs sweep
//    them with snake_item().  All CTAs work on different heads at once.
//  - pairs: a unit is one head and two key tiles t and n_kv - 1 - t, taken
//    one after the other by the same CTA.  Under a causal mask every pair
//    has the same number of steps (n_q + 1), so the units can be numbered
//    head major without unbalancing the CTAs, and the CTAs in flight cover
//    only about 148 / (n_kv / 2) heads: their Q, dO and FP32 dQ accumulator
//    then stay in the L2 instead of being streamed again for every key tile.
//    The host chooses it (a separate kernel instantiation) when the heads the
//    default order keeps in flight would not fit in the L2 together.
template <bool kPairs>
struct BwdSched {
  int rnd, sub, item, per_head, n_units;
  __device__ __forceinline__ explicit BwdSched(const BwdParams& p) : rnd(0), sub(0), item(snake_item(0)) {
    per_head = kPairs ? (p.n_kv + 1) / 2 : p.n_kv;
    n_units = per_head * p.BH;
  }
  __device__ __forceinline__ bool valid() const { return item < n_units; }
  __device__ __forceinline__ BwdItem get(const BwdParams& p) const {
    if constexpr (!kPairs) {
      return bwd_item_at(p, item % p.BH, item / p.BH);
    } else {
      const int pp = item % per_head;
      return bwd_item_at(p, item / per_head, sub ? p.n_kv - 1 - pp : pp);
    }
  }
  __device__ __forceinline__ void next(const BwdParams& p) {
    if constexpr (kPairs) {
      if (sub == 0 && 2 * (item % per_head) + 1 != p.n_kv) {   // a lone middle tile has no second
        sub = 1;
        return;
      }
      sub = 0;
    }
    item = snake_item(++rnd);
  }
};

// The steps of an item in order: query tile qt of batch*query-head bh_q,
// query tiles innermost.  Advanced once per step, without divisions.
struct BwdSteps {
  int qt, bh_q, q_first, q_end;
  __device__ __forceinline__ BwdSteps(const BwdParams& p, const BwdItem& w) {
    const int hkv = p.H / p.group;
    q_first = w.i_start;
    q_end = w.i_start + w.n_it_head;
    qt = q_first;
    bh_q = (w.bh / hkv) * p.H + (w.bh % hkv) * p.group;
  }
  __device__ __forceinline__ void next() {
    if (++qt == q_end) {
      qt = q_first;
      ++bh_q;
    }
  }
};

// Roles (16 warps):
//   warps 0-7   key-row math; warp w owns keys 32*(w%4).. (TMEM lane quarter
//               w%4) and queries 64*(w/4).. of each tile: P^T, dS^T
//   warps 8-11  dQ drain (thread r owns query r; TMA reduce-add of 32 x 32
//               FP32 boxes staged in shared memory) and the dK/dV epilogue
//               (d = 64: through the same staging boxes and TMA stores)
//   warp  12    producer: K, V per item; Q_i (TMA) plus LSE_i, D_i per step,
//               up to kQStages steps ahead
//   warp  14    producer: dO_i (TMA), independent of the Q ring
//   warp  13    TMEM allocator + tcgen05.mma issuer (the whole warp runs the
//               issuing loop; one elected lane executes each instruction)
//   warp  15    idle (completes the fourth warpgroup)
// MMA order per query tile i (the tensor core runs the next tile's S while
// the CUDA cores form dS_i, and dK_i, dQ_i, dP_{i+1} while they form P_{i+1}):
//   dV_i += P_bar_i^T dO_i | S_{i+1} | dK_i += dS_i^T Q_i | dQ_i = dS_i K | dP_{i+1}
// Barrier phases run on per-CTA counters, so items follow one another without
// re-initialisation: `g` counts query-tile steps, `n_done` counts items.
// E: the element format (ElemBF16 or ElemF16) of Q, K, V, dO, dK, dV and of
// the P_bar and dS operands.  kPairs: the head-major pair schedule (BwdSched).
template <int D, typename E = ElemBF16, bool kPairs = false>
__global__ void __launch_bounds__(512, 1)
    fa_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                  const __grid_constant__ CUtensorMap tm_dq, const __grid_constant__ CUtensorMap tm_dk,
                  const __grid_constant__ CUtensorMap tm_dv, const BwdParams p) {
  using L = BwdLayout<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* kv_full = bars;        // [2]
  uint64_t* kv_empty = bars + 2;   // [2]
  uint64_t* do_full = bars + 4;    // [2]
  uint64_t* do_empty = bars + 6;   // [2]
  uint64_t* s_full = bars + 8;
  uint64_t* p_full = bars + 9;
  uint64_t* dp_full = bars + 10;
  uint64_t* ds_full = bars + 11;
  uint64_t* dq_full = bars + 12;
  uint64_t* dq_free = bars + 13;
  uint64_t* dkv_done = bars + 14;
  uint64_t* dkv_free = bars + 15;
  uint64_t* mma_done = bars + 17;
  uint64_t* q_full = bars + 18;    // [kQStages]
  uint64_t* q_empty = bars + 21;   // [kQStages]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 24);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* stats = reinterpret_cast<float*>(smem + L::kStatOff);   // [stage][-lse2 | dsum][128]

  // The 128-byte swizzle needs 1 KB aligned tiles; the layout has no room to
  // realign, so a misaligned dynamic shared-memory base is reported, not used.
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) atomicExch(p.dev_error, kDevErrSmemAlign);
    return;
  }
  const int warp = int(warp_id());
  const int lane = int(lane_id());

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
      mbar_init(&do_full[s], 1);
      mbar_init(&do_empty[s], 1);
    }
    for (int s = 0; s < L::kQStages; ++s) {
      mbar_init(&q_full[s], 2);      // the Q tile's bytes, and the LSE/D rows in shared memory
      mbar_init(&q_empty[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(p_full, 256);
    mbar_init(dp_full, 1);
    mbar_init(ds_full, 256);
    mbar_init(dq_full, 1);
    mbar_init(dq_free, 128);
    mbar_init(dkv_done, 1);
    mbar_init(dkv_free, 128);
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 13) {
    tmem_alloc(tmem_slot, L::kTmemCols);
    tmem_relinquish();
  }
  if (warp == 12 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_do);
    tma_prefetch_desc(&tm_dq);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // Set-up above touched no global memory.  Launched right after the
  // preprocess kernel (after_pre), which let this kernel start only once every
  // kernel before it had finished, Q, K, V, dO and LSE are complete here and
  // only D and the zeroed dQ accumulator are not: then only the threads that
  // read D (the Q producer) or write global memory (the dQ drain and the
  // dK/dV epilogue) wait for the preprocess, and the K, V, Q and dO loads and
  // the first S and dP MMAs overlap its end.  Otherwise every thread waits.
  if (!p.after_pre) grid_dep_wait();
  grid_dep_launch();
  const Watchdog wd{abort_flag, p.dev_error};

  if (warp >= 12) {
    // Producer and MMA warps need few registers; give them back first.
    regs_set<L::kOtherRegs, L::kLaunchRegs>();
    if (warp == 12) {
      // ----------------------------------------------------------- producer
      const uint64_t pol_kv = l2_policy_evict_first();
      const uint64_t pol_q = l2_policy_evict_last();
      const float kLog2e = 1.4426950408889634f;
      uint32_t g = 0;        // query-tile steps loaded
      uint32_t n_done = 0;   // items started
      bool ok = true;
      bool dep_done = false;
      for (BwdSched<kPairs> sc(p); ok && sc.valid(); sc.next(p), ++n_done) {
        const BwdItem w = sc.get(p);
        const uint32_t ks = n_done % L::kKVStages;
        ok = __all_sync(0xffffffffu, mbar_wait(&kv_empty[ks], ((n_done / L::kKVStages) & 1) ^ 1, wd));
        if (!ok) break;
        if (lane == 0) {
          uint8_t* sk = smem + L::kKVOff + ks * 2 * L::kTileBytes;
          mbar_arrive_expect_tx(&kv_full[ks], uint32_t(2 * L::kTileBytes));
          for (int s = 0; s < L::kSub; ++s) {
            tma_load_3d(sk + s * L::kSubBytes, &tm_k, &kv_full[ks], s * 64, w.key0, w.bh, pol_kv);
            tma_load_3d(sk + L::kTileBytes + s * L::kSubBytes, &tm_v, &kv_full[ks], s * 64, w.key0, w.bh, pol_kv);
          }
        }
        BwdSteps sp(p, w);
        for (int it = 0; it < w.n_it; ++it, ++g, sp.next()) {
          const uint32_t st = g % L::kQStages;
          const int q0 = sp.qt * 128;
          ok = __all_sync(0xffffffffu, mbar_wait(&q_empty[st], ((g / L::kQStages) & 1) ^ 1, wd));
          if (!ok) break;
          // the Q tile first, so that its load overlaps the LSE/D reads below
          if (lane == 0) {
            mbar_arrive_expect_tx(&q_full[st], uint32_t(L::kTileBytes));
            for (int s = 0; s < L::kSub; ++s)
              tma_load_3d(smem + L::kQOff + st * L::kTileBytes + s * L::kSubBytes, &tm_q, &q_full[st], s * 64, q0,
                          sp.bh_q, pol_q);
          }
          if (!dep_done) {                     // D comes from the preprocess kernel
            grid_dep_wait();
            dep_done = true;
          }
          float* nlse = stats + st * 256;
          float* dd = nlse + 128;
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int r = lane * 4 + u;
            const int row = q0 + r;
            const bool in = row < p.N;
            // rows past N: P = 2^(-inf) = 0 and D = 0, so they add nothing
            nlse[r] = in ? -p.lse[size_t(sp.bh_q) * p.N + row] * kLog2e : -__int_as_float(0x7f800000);
            dd[r] = in ? p.dsum[size_t(sp.bh_q) * p.N + row] : 0.f;
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&q_full[st]);   // second arrival: the rows are in shared memory
        }
      }
    } else if (warp == 14) {
      // ------------------------------------------------------- dO producer
      const uint64_t pol_q = l2_policy_evict_last();
      uint32_t g = 0;
      bool ok = true;
      for (BwdSched<kPairs> sc(p); ok && sc.valid(); sc.next(p)) {
        const BwdItem w = sc.get(p);
        BwdSteps sp(p, w);
        for (int it = 0; it < w.n_it; ++it, ++g, sp.next()) {
          const int q0 = sp.qt * 128;
          // dO_i: with a single buffer it is refilled once dV_{i-1} has read it
          const uint32_t sd = g % L::kDOStages;
          ok = __all_sync(0xffffffffu, mbar_wait(&do_empty[sd], ((g / L::kDOStages) & 1) ^ 1, wd));
          if (!ok) break;
          if (lane == 0) {
            mbar_arrive_expect_tx(&do_full[sd], uint32_t(L::kTileBytes));
            for (int s = 0; s < L::kSub; ++s)
              tma_load_3d(smem + L::kDOOff + sd * L::kTileBytes + s * L::kSubBytes, &tm_do, &do_full[sd], s * 64,
                          q0, sp.bh_q, pol_q);
          }
          __syncwarp();
        }
      }
    } else if (warp == 13) {
      // ---------------------------------------------------------- MMA issuer
      // The whole warp runs this loop (warp-uniform operands and waits); one
      // elected lane executes each tcgen05.mma and tcgen05.commit.
      {
        constexpr uint32_t kIdS = make_idesc(128, 128, 0, 0, E::kMmaFmt);   // K Q^T, V dO^T: K-major operands
        constexpr uint32_t kIdAcc = make_idesc(128, D, 0, 1, E::kMmaFmt);   // TMEM A x MN-major B (dV, dK)
        constexpr uint32_t kIdDQ = make_idesc(128, D, 1, 1, E::kMmaFmt);    // dS (MN-major) x K (MN-major)
        // Descriptors as 32-bit low halves with one shared high half (every
        // operand has a 1024-byte stride): this warp shares its issue slots
        // with the busiest warps of the CTA, so each MMA costs it only an add.
        // K-major operands use a leading byte offset of 16, MN-major ones the
        // distance between 64-wide blocks.
        constexpr uint32_t kHi = sdesc_hi(1024);
        constexpr uint32_t kLboMN = uint32_t(L::kSubBytes >> 4) << 16;
        constexpr uint32_t kLboK = uint32_t(16 >> 4) << 16;
        const uint32_t ds_lo = sdesc_lo(smem_u32(smem + L::kDSOff), L::kSubBytes);
        auto kmajor_mma = [&](uint32_t d_tm, uint32_t a_lo, uint32_t b_lo) {   // low halves without LBO
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const uint32_t off = ((k >> 2) * L::kSubBytes + (k & 3) * 32) >> 4;
            umma_ss_lh_warp(d_tm, (a_lo + off) | kLboK, (b_lo + off) | kLboK, kHi, kIdS, k > 0 ? 1u : 0u);
          }
        };
        // start-address halves (address >> 4) of each buffer
        auto q_of = [&](uint32_t gg) {
          return (smem_u32(smem + L::kQOff) >> 4) + (gg % L::kQStages) * (L::kTileBytes >> 4);
        };
        auto do_of = [&](uint32_t gg) {
          return (smem_u32(smem + L::kDOOff) >> 4) + (gg % L::kDOStages) * (L::kTileBytes >> 4);
        };
        auto wait_q = [&](uint32_t gg) {
          return __all_sync(0xffffffffu, mbar_wait(&q_full[gg % L::kQStages], (gg / L::kQStages) & 1, wd));
        };
        auto wait_do = [&](uint32_t gg) {
          return __all_sync(0xffffffffu, mbar_wait(&do_full[gg % L::kDOStages], (gg / L::kDOStages) & 1, wd));
        };
        // K and V of the item started n items ago (start-address halves)
        auto k_of = [&](uint32_t n) {
          return (smem_u32(smem + L::kKVOff) >> 4) + (n % L::kKVStages) * (2 * L::kTileBytes >> 4);
        };
        uint32_t g = 0;        // query-tile steps issued
        uint32_t n_done = 0;   // items started
        bool ok = true;
        // d = 64 holds two items' K and V: the next item's first S^T and dP^T
        // are issued during this item's last step (as within an item), so
        // the compute warps do not wait for them at the item boundary
        bool first_issued = false;
        for (BwdSched<kPairs> sc(p); ok && sc.valid(); sc.next(p), ++n_done) {
          const BwdItem w = sc.get(p);
          const uint32_t ks = n_done % L::kKVStages;
          const uint32_t sk = k_of(n_done);
          const uint32_t sv = sk + (L::kTileBytes >> 4);
          BwdSched<kPairs> nx = sc;
          nx.next(p);
          const bool prefetch_next = !L::kWide && nx.valid();
          const uint32_t nsk = k_of(n_done + 1);
          const uint32_t nsv = nsk + (L::kTileBytes >> 4);
          if (!first_issued) {
            if (!(ok = __all_sync(0xffffffffu, mbar_wait(&kv_full[ks], (n_done / L::kKVStages) & 1, wd)) && wait_q(g) && wait_do(g))) break;
            tc_fence_after();
            kmajor_mma(tmem + L::kTmS, sk, q_of(g));     // S^T = K Q^T of the item's first query tile
            umma_commit_warp(s_full);
            if (L::kWide && g > 0) {                      // the previous dQ shares the dP^T columns
              if (!(ok = __all_sync(0xffffffffu, mbar_wait(dq_free, (g - 1) & 1, wd)))) break;
              tc_fence_after();
            }
            kmajor_mma(tmem + L::kTmDP, sv, do_of(g));   // dP^T = V dO^T
            umma_commit_warp(dp_full);
          }
          first_issued = false;
          // the first dV/dK MMA of an item overwrites the accumulators: the
          // previous item's epilogue must have read them
          if (!(ok = __all_sync(0xffffffffu, mbar_wait(dkv_free, (n_done & 1) ^ 1, wd)))) break;
          for (int it = 0; ok && it < w.n_it; ++it, ++g) {
            const uint32_t sq = q_of(g);
            const uint32_t sdo = do_of(g);
            if (!(ok = __all_sync(0xffffffffu, mbar_wait(p_full, g & 1, wd)))) break;
            tc_fence_after();
#pragma unroll
            for (int k = 0; k < 8; ++k)                 // dV += P_bar^T dO_i
              umma_ts_lh_warp(tmem + L::kTmDV, tmem + L::pt_col(k), (sdo + k * (2048 >> 4)) | kLboMN, kHi, kIdAcc,
                         (it > 0 || k > 0) ? 1u : 0u);
            umma_commit_warp(&do_empty[g % L::kDOStages]);   // dP_i and dV_i were the readers of dO_i
            if (it + 1 < w.n_it) {                      // S^T_{i+1}
              if (!(ok = wait_q(g + 1))) break;
              tc_fence_after();
              kmajor_mma(tmem + L::kTmS, sk, q_of(g + 1));
              umma_commit_warp(s_full);
            } else if (prefetch_next) {                 // the next item's first S^T, with its K
              if (!(ok = __all_sync(0xffffffffu, mbar_wait(&kv_full[(n_done + 1) % L::kKVStages], ((n_done + 1) / L::kKVStages) & 1, wd)) &&
                         wait_q(g + 1)))
                break;
              tc_fence_after();
              kmajor_mma(tmem + L::kTmS, nsk, q_of(g + 1));
              umma_commit_warp(s_full);
            }
            if (!(ok = __all_sync(0xffffffffu, mbar_wait(ds_full, g & 1, wd)))) break;
            tc_fence_after();
#pragma unroll
            for (int k = 0; k < 8; ++k)                 // dK += dS^T Q_i
              umma_ts_lh_warp(tmem + L::kTmDK, tmem + L::dst_col(k), (sq + k * (2048 >> 4)) | kLboMN, kHi, kIdAcc,
                         (it > 0 || k > 0) ? 1u : 0u);
            if (!L::kWide && g > 0) {                   // the drain has read dQ of the previous step
              if (!(ok = __all_sync(0xffffffffu, mbar_wait(dq_free, (g - 1) & 1, wd)))) break;
              tc_fence_after();
            }
#pragma unroll
            for (int k = 0; k < 8; ++k)                 // dQ_i = dS K
              umma_ss_lh_warp(tmem + L::kTmDQ, ds_lo + k * (2048 >> 4), (sk + k * (2048 >> 4)) | kLboMN, kHi, kIdDQ,
                         k > 0 ? 1u : 0u);
            umma_commit_warp(dq_full);
            umma_commit_warp(&q_empty[g % L::kQStages]);
            if (it + 1 < w.n_it) {                      // dP^T_{i+1}
              if (L::kWide) {                           // dQ_i shares the dP^T columns
                if (!(ok = __all_sync(0xffffffffu, mbar_wait(dq_free, g & 1, wd)))) break;
                tc_fence_after();
              }
              if (!(ok = wait_do(g + 1))) break;
              tc_fence_after();
              kmajor_mma(tmem + L::kTmDP, sv, do_of(g + 1));
              umma_commit_warp(dp_full);
            } else if (prefetch_next) {                 // the next item's first dP^T, with its V
              if (!(ok = wait_do(g + 1))) break;
              tc_fence_after();
              kmajor_mma(tmem + L::kTmDP, nsv, do_of(g + 1));
              umma_commit_warp(dp_full);
              first_issued = true;
            }
          }
          umma_commit_warp(&kv_empty[ks]);                   // K and V of this item are no longer read
          umma_commit_warp(dkv_done);                        // dK, dV of this item are final
        }
        umma_commit_warp(mma_done);
        __all_sync(0xffffffffu, mbar_wait(mma_done, 0, wd));
      }
      __syncwarp();
    }
  } else if (warp < 8) {
    regs_set<L::kComputeRegs, L::kLaunchRegs>();
    // ------------------------------------------------------- key-row math
    const int quarter = warp & 3;
    const int half = warp >> 2;                      // queries 64*half .. +63
    const int kr = quarter * 32 + lane;              // key within the tile
    const uint32_t lane_base = uint32_t(quarter * 32) << 16;
    const uint32_t t_s = tmem + lane_base + L::kTmS + 64 * half;
    const uint32_t t_dp = tmem + lane_base + L::kTmDP + 64 * half;
    const uint32_t t_pt = tmem + lane_base + (L::kWide ? L::kTmS + 64 * half : L::kTmPT + 32 * half);
    uint8_t* ds_row = smem + L::kDSOff + half * L::kSubBytes + kr * 128;
    const uint64_t c2 = f2_pack(p.scale_log2, p.scale_log2);
    uint32_t g = 0;
    bool ok = true;
    for (BwdSched<kPairs> sc(p); ok && sc.valid(); sc.next(p)) {
      const BwdItem w = sc.get(p);
      const bool key_in = w.key0 + kr < p.N;
      BwdSteps sp(p, w);
      for (int it = 0; it < w.n_it; ++it, ++g, sp.next()) {
        const uint32_t st = g % L::kQStages;
        const int qt = sp.qt;
        const float* nlse = stats + st * 256 + 64 * half;
        const float* dd = stats + st * 256 + 128 + 64 * half;
        // q_full publishes this stage's LSE/D (written by the producer's lanes)
        ok = __all_sync(0xffffffffu, mbar_wait(&q_full[st], (g / L::kQStages) & 1, wd)) &&
             __all_sync(0xffffffffu, mbar_wait(s_full, g & 1, wd));
        if (!ok) break;
        tc_fence_after();
        // P^T: P[q] = 2^(S*scale_log2 - LSE2[q]); masked entries are 0
        uint32_t pk[32];
        {
          uint32_t r[2][32];
          tmem_ld32(t_s, r[0]);
          tmem_ld32(t_s + 32, r[1]);
          tmem_ld_wait(r[0]);
          tmem_ld_wait(r[1]);
          const bool diag = p.causal && qt == w.kv_tile;
          if (!__any_sync(0xffffffffu, !key_in || diag)) {   // no masked entry in this warp
#pragma unroll
            for (int j = 0; j < 16; ++j) {             // 4 queries per shared-memory load of -LSE2
              const float4 nl = *reinterpret_cast<const float4*>(nlse + 4 * j);
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                const int i = 2 * j + h;               // pair of queries 2i, 2i+1 of this half
                float x0, x1;
                f2_unpack(f2_fma(f2_pack(__uint_as_float(r[i >> 4][(2 * i) & 31]),
                                         __uint_as_float(r[i >> 4][(2 * i + 1) & 31])),
                                 c2, h ? f2_pack(nl.z, nl.w) : f2_pack(nl.x, nl.y)),
                          x0, x1);
                pk[i] = E::pack(ex2(x0), ex2(x1));
              }
            }
          } else {
            // masked keys (past N) and, on the diagonal tile, queries before
            // the key: the exponent is set to -inf, so P = 0 (selected
            // alongside the exponentials; a separate pass that cleared the
            // packed halves afterwards cost ~1600 cycles per diagonal step)
            const int lim = key_in ? (diag ? kr - 64 * half : 0) : 64;   // queries q < lim are masked
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const float4 nl = *reinterpret_cast<const float4*>(nlse + 4 * j);
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                const int i = 2 * j + h;
                float x0, x1;
                f2_unpack(f2_fma(f2_pack(__uint_as_float(r[i >> 4][(2 * i) & 31]),
                                         __uint_as_float(r[i >> 4][(2 * i + 1) & 31])),
                                 c2, h ? f2_pack(nl.z, nl.w) : f2_pack(nl.x, nl.y)),
                          x0, x1);
                x0 = (2 * i < lim) ? -__int_as_float(0x7f800000) : x0;
                x1 = (2 * i + 1 < lim) ? -__int_as_float(0x7f800000) : x1;
                pk[i] = E::pack(ex2(x0), ex2(x1));
              }
            }
          }
        }
        // No wait before overwriting P_bar^T: dV of the previous step, its
        // last reader, was issued before this step's S^T, and the tensor core
        // completes one thread's MMAs in order, so s_full implies it is done.
        {
          uint32_t wv[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) wv[i] = pk[i];
          tmem_st16(t_pt, wv);
#pragma unroll
          for (int i = 0; i < 16; ++i) wv[i] = pk[16 + i];
          tmem_st16(t_pt + 16, wv);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(p_full);

        if (!(ok = __all_sync(0xffffffffu, mbar_wait(dp_full, g & 1, wd)))) break;
        tc_fence_after();
        // dS^T = P_bar * (dP - D[q])
        uint32_t dsw[32];
        {
          uint32_t r[2][32];
          tmem_ld32(t_dp, r[0]);
          tmem_ld32(t_dp + 32, r[1]);
          tmem_ld_wait(r[0]);
          tmem_ld_wait(r[1]);
#pragma unroll
          for (int j = 0; j < 16; ++j) {               // 4 queries per shared-memory load of D
            const float4 d4 = *reinterpret_cast<const float4*>(dd + 4 * j);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int i = 2 * j + h;
              const float2 pp = E::unpack(pk[i]);
              const uint64_t dq2 = h ? f2_pack(d4.z, d4.w) : f2_pack(d4.x, d4.y);
              const uint64_t dp2 = f2_pack(__uint_as_float(r[i >> 4][(2 * i) & 31]),
                                           __uint_as_float(r[i >> 4][(2 * i + 1) & 31]));
              float y0, y1;
              f2_unpack(f2_mul(f2_fma(dq2, f2_pack(-1.f, -1.f), dp2), f2_pack(pp.x, pp.y)), y0, y1);
              dsw[i] = E::pack(y0, y1);
            }
          }
        }
        {
          uint32_t wv[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) wv[i] = dsw[i];
          tmem_st16(t_dp, wv);
#pragma unroll
          for (int i = 0; i < 16; ++i) wv[i] = dsw[16 + i];
          tmem_st16(t_dp + 16, wv);
        }
        // dS into shared memory for dQ = dS K: MN-major, 128-byte swizzle.
        // dQ of the previous step, its last reader, was issued before this
        // step's dP^T, so dp_full already implied that it is done.
#pragma unroll
        for (int c16 = 0; c16 < 8; ++c16) {
          uint4* dst = reinterpret_cast<uint4*>(ds_row + ((c16 ^ (kr & 7)) << 4));
          *dst = make_uint4(dsw[c16 * 4], dsw[c16 * 4 + 1], dsw[c16 * 4 + 2], dsw[c16 * 4 + 3]);
        }
        fence_proxy_async_smem();
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(ds_full);
      }
    }
  } else {
    regs_set<L::kDrainRegs, L::kLaunchRegs>();
    grid_dep_wait();                                   // the preprocess zeroes the dQ accumulator
    // ------------------------------------------- dQ drain and dK/dV epilogue
    const int wq = warp & 3;
    const int rr = wq * 32 + lane;                   // query row (dQ) / key row (dK, dV)
    const uint32_t lane_base = uint32_t(wq * 32) << 16;
    const uint32_t t_dq = tmem + lane_base + L::kTmDQ;
    uint8_t* stage = smem + L::kDQStageOff + wq * 2 * L::kStageBox;
    uint32_t box_seq = 0;
    uint32_t g = 0;
    uint32_t n_done = 0;
    bool ok = true;
    for (BwdSched<kPairs> sc(p); ok && sc.valid(); sc.next(p), ++n_done) {
      const BwdItem w = sc.get(p);
      BwdSteps sp(p, w);
      for (int it = 0; it < w.n_it; ++it, ++g, sp.next()) {
        ok = __all_sync(0xffffffffu, mbar_wait(dq_full, g & 1, wd));
        if (!ok) break;
        tc_fence_after();
        // TMEM -> swizzled 32 x 32 FP32 box in shared memory -> TMA reduce-add
        // into the FP32 accumulator (rows past N are dropped by the TMA unit)
#pragma unroll
        for (int c2 = 0; c2 < D / 64; ++c2) {          // two 32-column chunks per TMEM wait: dQ's
                                                       // columns are released sooner (d = 128: dP waits on them)
          uint32_t r[2][32];
          tmem_ld32(t_dq + (2 * c2) * 32, r[0]);
          tmem_ld32(t_dq + (2 * c2 + 1) * 32, r[1]);
          tmem_ld_wait(r[0]);
          tmem_ld_wait(r[1]);
          if (c2 == D / 64 - 1) {                      // dQ is in registers: its TMEM may be reused
            tc_fence_before();
            mbar_arrive(dq_free);
          }
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int c = 2 * c2 + h;
            uint8_t* box = stage + (box_seq & 1) * L::kStageBox;
            if (lane == 0) bulk_wait_read<1>();        // the reduce issued from this box is done reading
            __syncwarp();
#pragma unroll
            for (int c16 = 0; c16 < 8; ++c16)
              *reinterpret_cast<uint4*>(box + lane * 128 + ((c16 ^ (lane & 7)) << 4)) =
                  make_uint4(r[h][4 * c16], r[h][4 * c16 + 1], r[h][4 * c16 + 2], r[h][4 * c16 + 3]);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_reduce_add_3d(&tm_dq, box, c * 32, sp.qt * 128 + wq * 32, sp.bh_q);
              bulk_commit();
            }
            ++box_seq;
          }
        }
      }
      if (!ok) break;
      // epilogue: dV and scale * dK of this item's keys, bf16
      ok = __all_sync(0xffffffffu, mbar_wait(dkv_done, n_done & 1, wd));
      if (!ok) break;
      tc_fence_after();
      const int key = w.key0 + rr;
      if constexpr (D == 64) {
        // dV and dK through this warp's two staging boxes (32 rows each, the
        // 128-byte swizzle) and one TMA store box each; rows past N are
        // dropped by the tensor maps.  dV goes into the box the next dQ drain
        // writes first, whose last reader is then the older of the two stores.
#pragma unroll
        for (int which = 0; which < 2; ++which) {
          const uint32_t t_src = tmem + lane_base + (which ? L::kTmDK : L::kTmDV);
          const float mul = which ? p.scale : 1.f;
          uint32_t r[2][32];
          tmem_ld32(t_src, r[0]);
          tmem_ld32(t_src + 32, r[1]);
          tmem_ld_wait(r[0]);
          tmem_ld_wait(r[1]);
          if (which == 1) {
            tc_fence_before();
            mbar_arrive(dkv_free);                   // the next item may overwrite dK, dV
          }
          uint8_t* box = stage + ((box_seq + which) & 1) * L::kStageBox;
          if (lane == 0) bulk_wait_read<1>();        // the group that last read this box is done reading
          __syncwarp();
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const int h = c >> 2, i0 = (c & 3) * 8;
            uint4 v;
            v.x = E::pack(__uint_as_float(r[h][i0 + 0]) * mul, __uint_as_float(r[h][i0 + 1]) * mul);
            v.y = E::pack(__uint_as_float(r[h][i0 + 2]) * mul, __uint_as_float(r[h][i0 + 3]) * mul);
            v.z = E::pack(__uint_as_float(r[h][i0 + 4]) * mul, __uint_as_float(r[h][i0 + 5]) * mul);
            v.w = E::pack(__uint_as_float(r[h][i0 + 6]) * mul, __uint_as_float(r[h][i0 + 7]) * mul);
            *reinterpret_cast<uint4*>(box + lane * 128 + ((c ^ (lane & 7)) << 4)) = v;
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_3d(which ? &tm_dk : &tm_dv, box, 0, w.key0 + wq * 32, w.bh);
            bulk_commit();
          }
        }
        box_seq += 2;
      } else {
  #pragma unroll
        for (int which = 0; which < 2; ++which) {
          const uint32_t t_src = tmem + lane_base + (which ? L::kTmDK : L::kTmDV);
          const float mul = which ? p.scale : 1.f;
          uint32_t ov[D / 2];
  #pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t r[32];
            tmem_ld32(t_src + c * 32, r);
            tmem_ld_wait(r);
  #pragma unroll
            for (int i = 0; i < 16; ++i)
              ov[c * 16 + i] = E::pack(__uint_as_float(r[2 * i]) * mul, __uint_as_float(r[2 * i + 1]) * mul);
          }
          if (which == 1) {
            tc_fence_before();
            mbar_arrive(dkv_free);                     // the next item may overwrite dK, dV
          }
          if (key < p.N) {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<typename E::T*>(which ? p.dk : p.dv) +
                                                  (size_t(w.bh) * p.N + key) * D);
  #pragma unroll
            for (int i = 0; i < D / 8; ++i) dst[i] = make_uint4(ov[4 * i], ov[4 * i + 1], ov[4 * i + 2], ov[4 * i + 3]);
          }
        }
      }
    }
    if (lane == 0) bulk_wait<0>();                     // every reduce-add has landed
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 13) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

}  // namespace fa
