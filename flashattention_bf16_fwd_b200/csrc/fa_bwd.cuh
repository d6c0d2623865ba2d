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
//                      accumulator with vector atomics
//   fa_bwd_dq_kernel   dQ = scale * accumulator -> bf16 (HBM-bound)
//
// fa_bwd_kernel warp roles (320 threads):
//   warps 0-3  key-row math: thread r owns key r (TMEM lane r); P^T, dS^T
//   warps 4-7  dQ drain (thread r owns query r of the tile) and the dK/dV
//              epilogue
//   warp  8    producer: K, V once; Q_i, dO_i (TMA) plus LSE_i, D_i per step
//   warp  9    TMEM allocator + tcgen05.mma issuer
// TMEM: S^T [0,128) (P_bar^T aliases [0,64)), dP^T [128,256) (dS^T aliases
// [128,192)), dV, dK, then dQ (d=64) or dQ aliasing dP^T (d=128).
#pragma once

#include "sm100.cuh"

namespace fa {

// D_i = sum_k dO_ik O_ik in FP32; also zeroes the FP32 dQ accumulator.
// Eight threads per row; each covers d/8 consecutive elements.
__global__ void __launch_bounds__(256) fa_bwd_pre_kernel(const __nv_bfloat16* __restrict__ o,
                                                         const __nv_bfloat16* __restrict__ dout,
                                                         float* __restrict__ dsum, float* __restrict__ dq_acc,
                                                         long long rows, int d) {
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
      const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
      const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&b);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 fa = __bfloat1622float2(a2[i]);
        const float2 fb = __bfloat1622float2(b2[i]);
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
__global__ void __launch_bounds__(256) fa_bwd_dq_kernel(const float* __restrict__ acc,
                                                        __nv_bfloat16* __restrict__ dq, float scale,
                                                        long long n8) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n8) return;
  const float4 a = reinterpret_cast<const float4*>(acc)[2 * i];
  const float4 b = reinterpret_cast<const float4*>(acc)[2 * i + 1];
  uint4 w;
  w.x = pack_bf16(a.x * scale, a.y * scale);
  w.y = pack_bf16(a.z * scale, a.w * scale);
  w.z = pack_bf16(b.x * scale, b.y * scale);
  w.w = pack_bf16(b.z * scale, b.w * scale);
  reinterpret_cast<uint4*>(dq)[i] = w;
}

struct BwdParams {
  const float* lse;     // [BH, N] natural log
  const float* dsum;    // [BH, N] D_i
  float* dq_acc;        // [BH, N, D] FP32
  __nv_bfloat16* dk;    // [BH, N, D]
  __nv_bfloat16* dv;    // [BH, N, D]
  int* dev_error;
  int BH, N, n_kv, causal;
  float scale, scale_log2;
};

template <int D>
struct BwdLayout {
  static constexpr int kSub = D / 64;
  static constexpr int kSubBytes = 128 * 64 * 2;
  static constexpr int kTileBytes = kSub * kSubBytes;
  static constexpr int kKOff = 0;
  static constexpr int kVOff = kTileBytes;
  static constexpr int kQOff = 2 * kTileBytes;             // 2 stages
  static constexpr int kDOOff = kQOff + 2 * kTileBytes;    // 2 stages
  static constexpr int kDSOff = kDOOff + 2 * kTileBytes;   // dS, [128 keys][128 queries] bf16, MN-major
  static constexpr int kStatOff = kDSOff + 2 * kSubBytes;  // 2 stages x (LSE*log2e, D) x 128 floats
  static constexpr int kBarOff = kStatOff + 2 * 2 * 128 * 4;
  static constexpr int kBytes = kBarOff + 256;
  static constexpr int kAlloc = kBytes;                    // base is 1 KB aligned by declaration
  static constexpr uint32_t kTmemCols = 512;
  static constexpr int kThreads = 320;
  static constexpr bool kDqAliasDp = (D == 128);
  static constexpr uint32_t kTmS = 0, kTmDP = 128, kTmDV = 256, kTmDK = 256 + D;
  static constexpr uint32_t kTmDQ = kDqAliasDp ? 128 : 256 + 2 * D;
};

template <int D>
__global__ void __launch_bounds__(320, 1)
    fa_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                  const BwdParams p) {
  using L = BwdLayout<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* kv_full = bars;
  uint64_t* q_full = bars + 1;    // [2]
  uint64_t* q_empty = bars + 3;   // [2]
  uint64_t* s_full = bars + 5;
  uint64_t* p_full = bars + 6;
  uint64_t* dp_full = bars + 7;
  uint64_t* ds_full = bars + 8;
  uint64_t* dq_full = bars + 9;
  uint64_t* dq_free = bars + 10;
  uint64_t* dkv_done = bars + 11;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 12);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* stats = reinterpret_cast<float*>(smem + L::kStatOff);   // [stage][lse2 | dsum][128]

  // The 128-byte swizzle needs 1 KB aligned tiles; the layout has no room to
  // realign, so a misaligned dynamic shared-memory base is reported, not used.
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) atomicExch(p.dev_error, kDevErrSmemAlign);
    return;
  }
  const int kv_tile = int(blockIdx.x) / p.BH;
  const int bh = int(blockIdx.x) % p.BH;
  const int key0 = kv_tile * 128;
  const int n_q = (p.N + 127) / 128;
  const int i_start = p.causal ? kv_tile : 0;
  const int n_it = n_q - i_start;
  const int warp = int(warp_id());
  const int lane = int(lane_id());

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&q_full[s], 1);
      mbar_init(&q_empty[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(p_full, 128);
    mbar_init(dp_full, 1);
    mbar_init(ds_full, 128);
    mbar_init(dq_full, 1);
    mbar_init(dq_free, 128);
    mbar_init(dkv_done, 1);
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
    tma_prefetch_desc(&tm_do);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const Watchdog wd{abort_flag, p.dev_error};

  if (warp == 8) {
    // ------------------------------------------------------------- producer
    const uint64_t pol_kv = l2_policy_evict_first();
    const uint64_t pol_q = l2_policy_evict_last();
    if (lane == 0) {
      mbar_arrive_expect_tx(kv_full, uint32_t(2 * L::kTileBytes));
      for (int s = 0; s < L::kSub; ++s) {
        tma_load_3d(smem + L::kKOff + s * L::kSubBytes, &tm_k, kv_full, s * 64, key0, bh, pol_kv);
        tma_load_3d(smem + L::kVOff + s * L::kSubBytes, &tm_v, kv_full, s * 64, key0, bh, pol_kv);
      }
    }
    const float kLog2e = 1.4426950408889634f;
    for (int it = 0; it < n_it; ++it) {
      const int st = it & 1;
      const int q0 = (i_start + it) * 128;
      if (!__all_sync(0xffffffffu, mbar_wait(&q_empty[st], ((it >> 1) & 1) ^ 1, wd))) break;
      float* lse2 = stats + st * 256;
      float* dd = lse2 + 128;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int r = lane * 4 + u;
        const int row = q0 + r;
        const bool in = row < p.N;
        lse2[r] = in ? p.lse[size_t(bh) * p.N + row] * kLog2e : __int_as_float(0x7f800000);
        dd[r] = in ? p.dsum[size_t(bh) * p.N + row] : 0.f;
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive_expect_tx(&q_full[st], uint32_t(2 * L::kTileBytes));
        for (int s = 0; s < L::kSub; ++s) {
          tma_load_3d(smem + L::kQOff + st * L::kTileBytes + s * L::kSubBytes, &tm_q, &q_full[st], s * 64, q0, bh,
                      pol_q);
          tma_load_3d(smem + L::kDOOff + st * L::kTileBytes + s * L::kSubBytes, &tm_do, &q_full[st], s * 64, q0,
                      bh, pol_q);
        }
      }
      __syncwarp();
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdS = make_idesc_bf16(128, 128, 0, 0);   // K Q^T, V dO^T: K-major operands
      constexpr uint32_t kIdAcc = make_idesc_bf16(128, D, 0, 1);   // TMEM A x MN-major B (dV, dK)
      constexpr uint32_t kIdDQ = make_idesc_bf16(128, D, 1, 1);    // dS (MN-major) x K (MN-major)
      const uint32_t sk = smem_u32(smem + L::kKOff);
      const uint32_t sv = smem_u32(smem + L::kVOff);
      const uint32_t sds = smem_u32(smem + L::kDSOff);
      auto kmajor_mma = [&](uint32_t d_tm, uint32_t a, uint32_t b) {
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t off = (k >> 2) * L::kSubBytes + (k & 3) * 32;
          umma_ss(d_tm, make_sdesc_sw128(a + off, 16, 1024), make_sdesc_sw128(b + off, 16, 1024), kIdS, k > 0);
        }
      };
      bool ok = mbar_wait(kv_full, 0, wd);
      for (int it = 0; ok && it < n_it; ++it) {
        const int st = it & 1;
        const uint32_t sq = smem_u32(smem + L::kQOff + st * L::kTileBytes);
        const uint32_t sdo = smem_u32(smem + L::kDOOff + st * L::kTileBytes);
        if (!(ok = mbar_wait(&q_full[st], (it >> 1) & 1, wd))) break;
        tc_fence_after();
        kmajor_mma(tmem + L::kTmS, sk, sq);            // S^T = K Q_i^T
        umma_commit(s_full);
        if (L::kDqAliasDp && it > 0) {                  // dQ_{i-1} shares columns with dP^T
          if (!(ok = mbar_wait(dq_free, (it - 1) & 1, wd))) break;
          tc_fence_after();
        }
        kmajor_mma(tmem + L::kTmDP, sv, sdo);          // dP^T = V dO_i^T
        umma_commit(dp_full);
        if (!(ok = mbar_wait(p_full, it & 1, wd))) break;
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < 8; ++k)                     // dV += P_bar^T dO_i
          umma_ts(tmem + L::kTmDV, tmem + L::kTmS + k * 8, make_sdesc_sw128(sdo + k * 2048, L::kSubBytes, 1024),
                  kIdAcc, (it > 0 || k > 0) ? 1u : 0u);
        if (!(ok = mbar_wait(ds_full, it & 1, wd))) break;
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < 8; ++k)                     // dK += dS^T Q_i
          umma_ts(tmem + L::kTmDK, tmem + L::kTmDP + k * 8, make_sdesc_sw128(sq + k * 2048, L::kSubBytes, 1024),
                  kIdAcc, (it > 0 || k > 0) ? 1u : 0u);
        if (!L::kDqAliasDp && it > 0) {
          if (!(ok = mbar_wait(dq_free, (it - 1) & 1, wd))) break;
          tc_fence_after();
        }
#pragma unroll
        for (int k = 0; k < 8; ++k)                     // dQ_i = dS K
          umma_ss(tmem + L::kTmDQ, make_sdesc_sw128(sds + k * 2048, L::kSubBytes, 1024),
                  make_sdesc_sw128(sk + k * 2048, L::kSubBytes, 1024), kIdDQ, k > 0 ? 1u : 0u);
        umma_commit(dq_full);
        umma_commit(&q_empty[st]);
      }
      umma_commit(dkv_done);
      mbar_wait(dkv_done, 0, wd);
    }
    __syncwarp();
  } else if (warp < 4) {
    // ------------------------------------------------------- key-row math
    const int kr = warp * 32 + lane;                 // key within the tile
    const int key = key0 + kr;
    const bool key_in = key < p.N;
    const uint32_t lane_base = uint32_t(warp * 32) << 16;
    const uint32_t t_s = tmem + lane_base + L::kTmS;
    const uint32_t t_dp = tmem + lane_base + L::kTmDP;
    uint8_t* ds_row = smem + L::kDSOff + kr * 128;
    for (int it = 0; it < n_it; ++it) {
      const int st = it & 1;
      const int qt = i_start + it;
      const float* lse2 = stats + st * 256;
      const float* dd = lse2 + 128;
      // q_full publishes this stage's LSE/D (written by the producer's lanes)
      if (!__all_sync(0xffffffffu, mbar_wait(&q_full[st], (it >> 1) & 1, wd))) break;
      if (!__all_sync(0xffffffffu, mbar_wait(s_full, it & 1, wd))) break;
      tc_fence_after();
      // P^T row: P[q] = 2^(S*scale_log2 - LSE2[q]); masked entries are 0
      uint32_t pk[64];
      const bool diag = p.causal && qt == kv_tile;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        tmem_ld32(t_s + c * 32, r);
        tmem_ld_wait(r);
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          const int q = c * 32 + i;
          float p0 = ex2(fmaf(__uint_as_float(r[i]), p.scale_log2, -lse2[q]));
          float p1 = ex2(fmaf(__uint_as_float(r[i + 1]), p.scale_log2, -lse2[q + 1]));
          if (!key_in || (diag && q < kr)) p0 = 0.f;
          if (!key_in || (diag && q + 1 < kr)) p1 = 0.f;
          pk[(c * 32 + i) >> 1] = pack_bf16(p0, p1);
        }
      }
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) w[i] = pk[c * 16 + i];
        tmem_st16(t_s + c * 16, w);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(p_full);

      if (!__all_sync(0xffffffffu, mbar_wait(dp_full, it & 1, wd))) break;
      tc_fence_after();
      // dS^T row = P_bar * (dP - D[q])
      uint32_t dk_w[64];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        tmem_ld32(t_dp + c * 32, r);
        tmem_ld_wait(r);
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          const int q = c * 32 + i;
          const float2 pp = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&pk[q >> 1]));
          const float d0 = pp.x * (__uint_as_float(r[i]) - dd[q]);
          const float d1 = pp.y * (__uint_as_float(r[i + 1]) - dd[q + 1]);
          dk_w[q >> 1] = pack_bf16(d0, d1);
        }
      }
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) w[i] = dk_w[c * 16 + i];
        tmem_st16(t_dp + c * 16, w);
      }
      // dS into shared memory for dQ = dS K: MN-major, 128-byte swizzle
      if (it > 0) {
        if (!__all_sync(0xffffffffu, mbar_wait(dq_full, (it - 1) & 1, wd))) break;
      }
#pragma unroll
      for (int ch = 0; ch < 16; ++ch) {
        const int blk = ch >> 3, c16 = ch & 7;
        uint4* dst = reinterpret_cast<uint4*>(ds_row + blk * L::kSubBytes + ((c16 ^ (kr & 7)) << 4));
        *dst = make_uint4(dk_w[ch * 4], dk_w[ch * 4 + 1], dk_w[ch * 4 + 2], dk_w[ch * 4 + 3]);
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(ds_full);
    }
  } else {
    // ------------------------------------------- dQ drain and dK/dV epilogue
    const int wq = warp & 3;
    const int rr = wq * 32 + lane;                   // query row (dQ) / key row (dK, dV)
    const uint32_t lane_base = uint32_t(wq * 32) << 16;
    const uint32_t t_dq = tmem + lane_base + L::kTmDQ;
    bool ok = true;
    for (int it = 0; it < n_it; ++it) {
      const int row = (i_start + it) * 128 + rr;
      ok = __all_sync(0xffffffffu, mbar_wait(dq_full, it & 1, wd));
      if (!ok) break;
      tc_fence_after();
      float4* dst = reinterpret_cast<float4*>(p.dq_acc + (size_t(bh) * p.N + row) * D);
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(t_dq + c * 32, r);
        tmem_ld_wait(r);
        if (row < p.N) {
#pragma unroll
          for (int i = 0; i < 8; ++i)
            atomicAdd(dst + c * 8 + i, make_float4(__uint_as_float(r[4 * i]), __uint_as_float(r[4 * i + 1]),
                                                   __uint_as_float(r[4 * i + 2]), __uint_as_float(r[4 * i + 3])));
        }
      }
      tc_fence_before();
      mbar_arrive(dq_free);
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(dkv_done, 0, wd));
    if (ok) {
      tc_fence_after();
      const int key = key0 + rr;
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        const uint32_t t_src = tmem + lane_base + (which ? L::kTmDK : L::kTmDV);
        const float mul = which ? p.scale : 1.f;
        __nv_bfloat16* out = (which ? p.dk : p.dv) + (size_t(bh) * p.N + key) * D;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(t_src + c * 32, r);
          tmem_ld_wait(r);
          uint32_t w[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            w[i] = pack_bf16(__uint_as_float(r[2 * i]) * mul, __uint_as_float(r[2 * i + 1]) * mul);
          if (key < p.N) {
            uint4* dst = reinterpret_cast<uint4*>(out + c * 32);
#pragma unroll
            for (int i = 0; i < 4; ++i) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

}  // namespace fa
