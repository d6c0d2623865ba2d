// fa_api.cu - the C ABI declared in include/fa_b200.h: argument checks, TMA
// tensor maps, launch configuration, and the device error flag.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>
#include <mutex>
#include <utility>

#include "../../include/fa_b200.h"
#include "fa_bwd.cuh"
#include "fa_fwd.cuh"
#include "fa_selftest.cuh"

namespace fa {

// Set by a kernel whose bounded wait expired; read and cleared by
// fa_check_device_error().
__device__ int g_dev_error = 0;

namespace {

constexpr int kMaxDevices = 64;

struct DeviceState {
  std::once_flag once;
  int status = FA_ERR_DEVICE;   // FA_OK once the device passed every check below
  int num_sms = 0;
  int* dev_error = nullptr;
};
DeviceState g_devices[kMaxDevices];

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode;
}

// Per-device set-up, done once with that device current: check the
// architecture, opt the kernels into large shared memory, and resolve the
// device address of the error flag.  Returns nullptr on failure; `why` (if
// given) receives FA_ERR_DEVICE or FA_ERR_BUILD.
DeviceState* device_state(int* why = nullptr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  DeviceState* st = &g_devices[dev];
  std::call_once(st->once, [st, dev] {
    cudaDeviceProp prop{};
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess || prop.major != 10) return;
    st->num_sms = prop.multiProcessorCount;
    void* addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_dev_error) != cudaSuccess) return;
    st->dev_error = static_cast<int*>(addr);
    bool ok = true;
    bool regs_ok = true;
    // Every kernel instantiation: large shared memory, and the register count
    // at launch that its setmaxnreg split assumes (a miscounted pool would stall
    // setmaxnreg.inc, so a build whose count differs is refused as FA_ERR_BUILD).
    auto setup = [&](auto kernel, int smem, int regs) {
      cudaFuncAttributes fattr{};
      ok &= cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) == cudaSuccess;
      ok &= cudaFuncGetAttributes(&fattr, kernel) == cudaSuccess;
      regs_ok &= fattr.numRegs == regs;
    };
    setup(fa_fwd_kernel<64, false, ElemBF16>, FwdLayout<64>::kAlloc, FwdLayout<64>::kLaunchRegs);
    setup(fa_fwd_kernel<128, false, ElemBF16>, FwdLayout<128>::kAlloc, FwdLayout<128>::kLaunchRegs);
    setup(fa_fwd_kernel<64, true, ElemBF16>, FwdLayout<64>::kAlloc, FwdLayout<64>::kLaunchRegs);
    setup(fa_fwd_kernel<128, true, ElemBF16>, FwdLayout<128>::kAlloc, FwdLayout<128>::kLaunchRegs);
    setup(fa_fwd_kernel<64, false, ElemF16>, FwdLayout<64>::kAlloc, FwdLayout<64>::kLaunchRegs);
    setup(fa_fwd_kernel<128, false, ElemF16>, FwdLayout<128>::kAlloc, FwdLayout<128>::kLaunchRegs);
    setup(fa_fwd_kernel<64, true, ElemF16>, FwdLayout<64>::kAlloc, FwdLayout<64>::kLaunchRegs);
    setup(fa_fwd_kernel<128, true, ElemF16>, FwdLayout<128>::kAlloc, FwdLayout<128>::kLaunchRegs);
    setup(fa_bwd_kernel<64, ElemBF16, false>, BwdLayout<64>::kAlloc, BwdLayout<64>::kLaunchRegs);
    setup(fa_bwd_kernel<128, ElemBF16, false>, BwdLayout<128>::kAlloc, BwdLayout<128>::kLaunchRegs);
    setup(fa_bwd_kernel<64, ElemF16, false>, BwdLayout<64>::kAlloc, BwdLayout<64>::kLaunchRegs);
    setup(fa_bwd_kernel<128, ElemF16, false>, BwdLayout<128>::kAlloc, BwdLayout<128>::kLaunchRegs);
    setup(fa_bwd_kernel<64, ElemBF16, true>, BwdLayout<64>::kAlloc, BwdLayout<64>::kLaunchRegs);
    setup(fa_bwd_kernel<128, ElemBF16, true>, BwdLayout<128>::kAlloc, BwdLayout<128>::kLaunchRegs);
    setup(fa_bwd_kernel<64, ElemF16, true>, BwdLayout<64>::kAlloc, BwdLayout<64>::kLaunchRegs);
    setup(fa_bwd_kernel<128, ElemF16, true>, BwdLayout<128>::kAlloc, BwdLayout<128>::kLaunchRegs);
    st->status = !ok ? FA_ERR_DEVICE : !regs_ok ? FA_ERR_BUILD : FA_OK;
  });
  if (st->status != FA_OK) {
    if (why) *why = st->status;
    return nullptr;
  }
  return st;
}

// device_state() for an entry point: the state, or the status to return.
#define FA_DEVICE_OR_RETURN(var)              \
  int var##_why = FA_ERR_DEVICE;              \
  DeviceState* var = device_state(&var##_why); \
  if (!var) return var##_why

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Every kernel is launched with programmatic stream serialisation: it may be
// scheduled while the previous kernel in the stream drains, runs its set-up
// (barriers, TMEM, descriptor prefetch), and waits in grid_dep_wait() before
// it touches global memory.
constexpr int kProgrammaticLaunch = 1;

template <typename... KArgs, typename... Args>
cudaError_t launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                   Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = kProgrammaticLaunch;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

int check_common(int B, int H, int N, int d, int causal, float scale) {
  if (d != 64 && d != 128) return FA_ERR_HEADDIM;
  if (B < 1 || H < 1 || N < 1) return FA_ERR_SHAPE;
  const long long total = (long long)B * H * N * d;
  if (total >= (1ll << 31)) return FA_ERR_SHAPE;
  if (causal != 0 && causal != 1) return FA_ERR_ARG;
  if (!std::isfinite(scale) || !(scale > 0.f)) return FA_ERR_ARG;
  return FA_OK;
}

// A [BH, N, D] bf16 tensor seen as 3-D (d, n, bh); boxes of 64 x box_rows x 1
// (128 for the loads the tcgen05 descriptors read, 32 for the forward's O
// stores, one per warp) with the 128-byte swizzle.  Loads read 0 past N; stores
// drop rows past N.
bool make_map(CUtensorMap* map, const void* base, int BH, int N, int D,
              CUtensorMapDataType dt = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, unsigned box_rows = 128) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {cuuint64_t(D), cuuint64_t(N), cuuint64_t(BH)};
  cuuint64_t strides[2] = {cuuint64_t(D) * 2, cuuint64_t(N) * D * 2};
  cuuint32_t box[3] = {64, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, dt, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The FP32 dQ accumulator [BH, N, D] as 3-D (d, n, bh) with 32 x 32 boxes and
// the 128-byte swizzle, for TMA reduce-add.
bool make_map_dq(CUtensorMap* map, const void* base, int BH, int N, int D) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {cuuint64_t(D), cuuint64_t(N), cuuint64_t(BH)};
  cuuint64_t strides[2] = {cuuint64_t(D) * 4, cuuint64_t(N) * D * 4};
  cuuint32_t box[3] = {32, 32, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Shift added to m on repeated-max rows (base-2 units): maps a maximum to 1 - 2^-8.
const double kDeltaLog2 = -std::log2(1.0 - 1.0 / 256.0);
// The same for fp16 P_bar: maps a maximum to 1 - 2^-11.
const double kDeltaLog2F16 = -std::log2(1.0 - 1.0 / 2048.0);

template <typename E>
constexpr CUtensorMapDataType map_type() {
  return E::kMmaFmt == 1 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
}

// H query heads share Hkv key/value heads (H == Hkv: ordinary attention).
int check_heads(int H, int Hkv) { return (Hkv >= 1 && Hkv <= H && H % Hkv == 0) ? FA_OK : FA_ERR_SHAPE; }

template <typename E>
int launch_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int32_t* ties, int32_t* one_hit,
               float* o_f32, int B, int H, int Hkv, int N, int d, int causal, float scale, int fix_mode,
               cudaStream_t stream) {
  constexpr bool kF16 = E::kMmaFmt == 0;
  if (!q || !k || !v || !o || !lse) return FA_ERR_NULL;
  int rc = check_common(B, H, N, d, causal, scale);
  if (rc != FA_OK) return rc;
  if ((rc = check_heads(H, Hkv)) != FA_OK) return rc;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(o_f32)) return FA_ERR_ALIGN;
  if (fix_mode < 0 || fix_mode > 5) return FA_ERR_FIXMODE;
  FA_DEVICE_OR_RETURN(st);
  const int BH = B * H;
  CUtensorMap mq, mk, mv, mo;
  constexpr CUtensorMapDataType dt = map_type<E>();
  if (!make_map(&mq, q, BH, N, d, dt) || !make_map(&mk, k, B * Hkv, N, d, dt) ||
      !make_map(&mv, v, B * Hkv, N, d, dt) || !make_map(&mo, o, BH, N, d, dt, 32))
    return FA_ERR_DEVICE;
  FwdParams prm{};
  prm.H = H;
  prm.group = H / Hkv;
  prm.o = static_cast<__nv_bfloat16*>(o);
  prm.lse = lse;
  prm.ties = ties;
  prm.one_hit = one_hit;
  prm.o_f32 = o_f32;
  prm.dev_error = st->dev_error;
  prm.BH = BH;
  prm.N = N;
  prm.n_pairs = (N + 255) / 256;
  prm.causal = causal;
  prm.scale_log2 = float(double(scale) * 1.4426950408889634);
  // shift on repeated-max rows per fix_mode, in base-2 units: 1 and 5 map the
  // maxima to the largest value below 1 of the P_bar format (1 - 2^-8 in bf16,
  // 1 - 2^-11 in fp16), 2 to 0.5, 3 to exp(-1/16); 0 and 4 keep the plain shift
  const double delta = (fix_mode == 1 || fix_mode == 5) ? (kF16 ? kDeltaLog2F16 : kDeltaLog2)
                       : fix_mode == 2                  ? 1.0
                       : fix_mode == 3                  ? 1.4426950408889634 / 16.0
                                                        : 0.0;
  prm.delta_log2 = float(delta);
  prm.fix_factor = float(std::exp2(-delta));
  prm.fix = (fix_mode == 1 || fix_mode == 2 || fix_mode == 3 || fix_mode == 5) ? 1 : 0;
  prm.self_norm = (fix_mode == 4) ? 1 : 0;
  prm.near = (fix_mode == 5) ? 1 : 0;
  const int n_items = prm.n_pairs * BH;
  const dim3 grid(unsigned(n_items < st->num_sms ? n_items : st->num_sms));
  // self-normalised or near-tie code, or a debug record
  const bool variants = fix_mode >= 4 || ties || one_hit || o_f32;
  auto kern = (d == 64) ? (variants ? fa_fwd_kernel<64, true, E> : fa_fwd_kernel<64, false, E>)
                        : (variants ? fa_fwd_kernel<128, true, E> : fa_fwd_kernel<128, false, E>);
  const int smem = (d == 64) ? FwdLayout<64>::kAlloc : FwdLayout<128>::kAlloc;
  const cudaError_t e = launch(kern, grid, dim3(FwdLayout<64>::kThreads), smem, stream, mq, mk, mv, mo, prm);
  return e == cudaSuccess ? FA_OK : FA_ERR_LAUNCH;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace
}  // namespace fa

using namespace fa;

extern "C" {

int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d,
           int causal, float scale, int fix_mode, void* stream) {
  return launch_fwd<ElemBF16>(q, k, v, o, lse, nullptr, nullptr, nullptr, B, H, H, N, d, causal, scale, fix_mode,
                              static_cast<cudaStream_t>(stream));
}

size_t fa_bwd_workspace_size(int B, int H, int N, int d) {
  if (check_common(B, H, N, d, 0, 1.f) != FA_OK) return 0;
  const size_t rows = size_t(B) * H * N;
  return align256(rows * d * sizeof(float)) + align256(rows * sizeof(float));
}

}  // extern "C"

namespace fa {
namespace {

// The backward's three launches for element format E.
template <typename E>
int pre_impl(const void* o, const void* dout, void* workspace, size_t workspace_bytes, int B, int H, int N, int d,
             void* stream) {
  if (!o || !dout) return FA_ERR_NULL;
  int rc = check_common(B, H, N, d, 0, 1.f);
  if (rc != FA_OK) return rc;
  if (!aligned16(o) || !aligned16(dout)) return FA_ERR_ALIGN;
  if (!workspace || !aligned16(workspace) || workspace_bytes < fa_bwd_workspace_size(B, H, N, d))
    return FA_ERR_WORKSPACE;
  FA_DEVICE_OR_RETURN(st);
  (void)st;
  const size_t rows = size_t(B) * H * N;
  float* dq_acc = static_cast<float*>(workspace);
  float* dsum = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + align256(rows * d * sizeof(float)));
  const int threads = 256;
  const long long blocks = ((long long)rows * 8 + threads - 1) / threads;
  using T = typename E::T;
  const cudaError_t e = launch(fa_bwd_pre_kernel<E>, dim3(unsigned(blocks)), dim3(threads), 0,
                               static_cast<cudaStream_t>(stream), static_cast<const T*>(o),
                               static_cast<const T*>(dout), dsum, dq_acc, (long long)rows, d);
  return e == cudaSuccess ? FA_OK : FA_ERR_LAUNCH;
}

// The backward main kernel for H query heads sharing Hkv key/value heads.
template <typename E>
int bwd_main_impl(const void* q, const void* k, const void* v, const float* lse, const void* dout, void* dk, void* dv,
                  void* workspace, size_t workspace_bytes, int B, int H, int Hkv, int N, int d, int causal,
                  float scale, void* stream, bool after_pre = false) {
  if (!q || !k || !v || !lse || !dout || !dk || !dv) return FA_ERR_NULL;
  int rc = check_common(B, H, N, d, causal, scale);
  if (rc != FA_OK) return rc;
  if ((rc = check_heads(H, Hkv)) != FA_OK) return rc;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dout) || !aligned16(dk) || !aligned16(dv))
    return FA_ERR_ALIGN;
  if (!workspace || !aligned16(workspace) || workspace_bytes < fa_bwd_workspace_size(B, H, N, d))
    return FA_ERR_WORKSPACE;
  FA_DEVICE_OR_RETURN(st);
  const int BH = B * H;
  const size_t rows = size_t(BH) * N;
  const int BHkv = B * Hkv;
  constexpr CUtensorMapDataType dt = map_type<E>();
  CUtensorMap mq, mk, mv, mdo, mdq, mdk, mdv;
  if (!make_map(&mq, q, BH, N, d, dt) || !make_map(&mk, k, BHkv, N, d, dt) || !make_map(&mv, v, BHkv, N, d, dt) ||
      !make_map(&mdo, dout, BH, N, d, dt) || !make_map_dq(&mdq, workspace, BH, N, d) ||
      !make_map(&mdk, dk, BHkv, N, d, dt, 32) || !make_map(&mdv, dv, BHkv, N, d, dt, 32))
    return FA_ERR_DEVICE;
  BwdParams prm{};
  prm.lse = lse;
  prm.dsum = reinterpret_cast<const float*>(static_cast<uint8_t*>(workspace) + align256(rows * d * sizeof(float)));
  prm.dq_acc = static_cast<float*>(workspace);
  prm.dk = dk;
  prm.dv = dv;
  prm.dev_error = st->dev_error;
  prm.BH = BHkv;   // work items run over the K/V heads
  // Head-major pairs of key tiles when the heads the default (key-tile major)
  // order keeps in flight would stream more than half the L2 together: each
  // K/V head streams Q and dO (2 bytes an element) and the FP32 dQ
  // accumulator of each of its H / Hkv query heads.
  const double per_head = 8.0 * N * d * (H / Hkv);
  const double in_flight = BHkv < st->num_sms ? BHkv : st->num_sms;
  const bool pairs = in_flight * per_head > 64.0 * (1 << 20);
  prm.H = H;
  prm.group = H / Hkv;
  prm.N = N;
  prm.n_kv = (N + 127) / 128;
  prm.causal = causal;
  prm.scale = scale;
  prm.scale_log2 = float(double(scale) * 1.4426950408889634);
  prm.after_pre = after_pre ? 1 : 0;
  const int n_items = prm.n_kv * BHkv;
  const dim3 grid(unsigned(n_items < st->num_sms ? n_items : st->num_sms));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  auto kern = (d == 64) ? (pairs ? fa_bwd_kernel<64, E, true> : fa_bwd_kernel<64, E, false>)
                        : (pairs ? fa_bwd_kernel<128, E, true> : fa_bwd_kernel<128, E, false>);
  const int smem = (d == 64) ? BwdLayout<64>::kAlloc : BwdLayout<128>::kAlloc;
  const cudaError_t e = launch(kern, grid, dim3(BwdLayout<64>::kThreads), smem, s, mq, mk, mv, mdo, mdq, mdk, mdv, prm);
  return e == cudaSuccess ? FA_OK : FA_ERR_LAUNCH;
}

template <typename E>
int finish_impl(void* dq, const void* workspace, size_t workspace_bytes, int B, int H, int N, int d, float scale,
                void* stream) {
  if (!dq) return FA_ERR_NULL;
  int rc = check_common(B, H, N, d, 0, scale);
  if (rc != FA_OK) return rc;
  if (!aligned16(dq)) return FA_ERR_ALIGN;
  if (!workspace || !aligned16(workspace) || workspace_bytes < fa_bwd_workspace_size(B, H, N, d))
    return FA_ERR_WORKSPACE;
  FA_DEVICE_OR_RETURN(st);
  (void)st;
  const long long n8 = (long long)B * H * N * d / 8;
  const int threads = 256;
  const cudaError_t e = launch(fa_bwd_dq_kernel<E>, dim3(unsigned((n8 + threads - 1) / threads)), dim3(threads), 0,
                               static_cast<cudaStream_t>(stream), static_cast<const float*>(workspace),
                               static_cast<typename E::T*>(dq), scale, n8);
  return e == cudaSuccess ? FA_OK : FA_ERR_LAUNCH;
}

template <typename E>
int bwd_impl(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dout, void* dq,
             void* dk, void* dv, void* workspace, size_t workspace_bytes, int B, int H, int Hkv, int N, int d,
             int causal, float scale, void* stream) {
  // Check everything up front so that an error leaves every output untouched.
  if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv) return FA_ERR_NULL;
  int rc = check_common(B, H, N, d, causal, scale);
  if (rc != FA_OK) return rc;
  if ((rc = check_heads(H, Hkv)) != FA_OK) return rc;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) || !aligned16(dq) ||
      !aligned16(dk) || !aligned16(dv))
    return FA_ERR_ALIGN;
  if (!workspace || !aligned16(workspace) || workspace_bytes < fa_bwd_workspace_size(B, H, N, d))
    return FA_ERR_WORKSPACE;
  FA_DEVICE_OR_RETURN(st);
  (void)st;
  rc = pre_impl<E>(o, dout, workspace, workspace_bytes, B, H, N, d, stream);
  if (rc != FA_OK) return rc;
  // launched right after the preprocess: it may start its input loads early
  rc = bwd_main_impl<E>(q, k, v, lse, dout, dk, dv, workspace, workspace_bytes, B, H, Hkv, N, d, causal, scale,
                        stream, true);
  if (rc != FA_OK) return rc;
  return finish_impl<E>(dq, workspace, workspace_bytes, B, H, N, d, scale, stream);
}

}  // namespace
}  // namespace fa

extern "C" {

int fa_bwd_preprocess(const void* o, const void* dout, void* workspace, size_t workspace_bytes, int B, int H,
                      int N, int d, void* stream) {
  return pre_impl<ElemBF16>(o, dout, workspace, workspace_bytes, B, H, N, d, stream);
}

int fa_bwd_main(const void* q, const void* k, const void* v, const float* lse, const void* dout, void* dk,
                void* dv, void* workspace, size_t workspace_bytes, int B, int H, int N, int d, int causal,
                float scale, void* stream) {
  return bwd_main_impl<ElemBF16>(q, k, v, lse, dout, dk, dv, workspace, workspace_bytes, B, H, H, N, d, causal,
                                 scale, stream);
}

int fa_bwd_finish(void* dq, const void* workspace, size_t workspace_bytes, int B, int H, int N, int d, float scale,
                  void* stream) {
  return finish_impl<ElemBF16>(dq, workspace, workspace_bytes, B, H, N, d, scale, stream);
}

int fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dout,
           void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes, int B, int H, int N, int d,
           int causal, float scale, void* stream) {
  return bwd_impl<ElemBF16>(q, k, v, o, lse, dout, dq, dk, dv, workspace, workspace_bytes, B, H, H, N, d, causal,
                            scale, stream);
}

// The general forward for element format `elem`, with the optional records.
static int fwd_elem(const void* q, const void* k, const void* v, void* o, float* lse, int32_t* ties,
                    int32_t* one_hit, float* o_f32, int B, int H, int Hkv, int N, int d, int causal, float scale,
                    int fix_mode, int elem, void* stream) {
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (elem == FA_ELEM_BF16)
    return launch_fwd<ElemBF16>(q, k, v, o, lse, ties, one_hit, o_f32, B, H, Hkv, N, d, causal, scale, fix_mode, s);
  if (elem == FA_ELEM_F16)
    return launch_fwd<ElemF16>(q, k, v, o, lse, ties, one_hit, o_f32, B, H, Hkv, N, d, causal, scale, fix_mode, s);
  return FA_ERR_ARG;
}

int fa_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Hkv, int N,
              int d, int causal, float scale, int fix_mode, int elem, void* stream) {
  return fwd_elem(q, k, v, o, lse, nullptr, nullptr, nullptr, B, H, Hkv, N, d, causal, scale, fix_mode, elem,
                  stream);
}

int fa_fwd_debug(const void* q, const void* k, const void* v, void* o, float* lse, int32_t* tie_count_out,
                 int32_t* one_hit_out, float* o_f32_out, int B, int H, int Hkv, int N, int d, int causal,
                 float scale, int fix_mode, int elem, void* stream) {
  if (!tie_count_out && !one_hit_out && !o_f32_out) return FA_ERR_NULL;
  return fwd_elem(q, k, v, o, lse, tie_count_out, one_hit_out, o_f32_out, B, H, Hkv, N, d, causal, scale, fix_mode,
                  elem, stream);
}

int fa_bwd_ex(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dout,
              void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes, int B, int H, int Hkv, int N,
              int d, int causal, float scale, int elem, void* stream) {
  if (elem == FA_ELEM_BF16)
    return bwd_impl<ElemBF16>(q, k, v, o, lse, dout, dq, dk, dv, workspace, workspace_bytes, B, H, Hkv, N, d,
                              causal, scale, stream);
  if (elem == FA_ELEM_F16)
    return bwd_impl<ElemF16>(q, k, v, o, lse, dout, dq, dk, dv, workspace, workspace_bytes, B, H, Hkv, N, d,
                             causal, scale, stream);
  return FA_ERR_ARG;
}

const char* fa_status_string(int status) {
  switch (status) {
    case FA_OK: return "ok";
    case FA_ERR_NULL: return "a required pointer is NULL";
    case FA_ERR_SHAPE: return "B, H or N < 1, or B*H*N*d >= 2^31";
    case FA_ERR_HEADDIM: return "head dimension d must be 64 or 128";
    case FA_ERR_ALIGN: return "a tensor base address is not 16-byte aligned";
    case FA_ERR_FIXMODE: return "fix_mode must be 0, 1, 2, 3, 4 or 5";
    case FA_ERR_WORKSPACE: return "workspace is NULL, misaligned or smaller than fa_bwd_workspace_size()";
    case FA_ERR_LAUNCH: return "the CUDA runtime refused a kernel launch";
    case FA_ERR_TIMEOUT: return "a kernel gave up on a bounded wait (device error flag set)";
    case FA_ERR_ARG:
      return "an argument is out of range: causal not 0 or 1, scale not finite and > 0, elem not an fa_elem "
             "value, or a watchdog timeout outside 1..1000000 us";
    case FA_ERR_DEVICE: return "no sm_100 device, or tensor-map encoding unavailable";
    case FA_ERR_BUILD:
      return "the library was compiled with a register count per thread that its kernels' register split "
             "does not expect (rebuild with the flags in build.py)";
    case FA_ERR_SCRATCH_LIMIT:
      return "fa_bwd_noalloc: fa_bwd_workspace_size() exceeds FA_BWD_NOALLOC_SCRATCH_BYTES (32 MiB)";
    default: return "unknown status";
  }
}

int fa_watchdog_selftest(unsigned timeout_us, void* stream) {
  if (timeout_us < 1 || timeout_us > 1000000) return FA_ERR_ARG;
  FA_DEVICE_OR_RETURN(st);
  const cudaError_t e = launch(fa_watchdog_selftest_kernel, dim3(1), dim3(64), 0, static_cast<cudaStream_t>(stream),
                               st->dev_error, uint64_t(timeout_us) * 1000ull);
  return e == cudaSuccess ? FA_OK : FA_ERR_LAUNCH;
}

int fa_check_device_error(void* stream) {
  FA_DEVICE_OR_RETURN(st);
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return FA_ERR_LAUNCH;
  int flag = 0;
  if (cudaMemcpy(&flag, st->dev_error, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return FA_ERR_LAUNCH;
  if (flag != kDevErrNone) {
    const int zero = 0;
    cudaMemcpy(st->dev_error, &zero, sizeof(int), cudaMemcpyHostToDevice);
    return flag == kDevErrTimeout ? FA_ERR_TIMEOUT : FA_ERR_DEVICE;
  }
  return FA_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// fa_bwd_noalloc: the backward pass for callers that cannot allocate device
// memory (an allocator owned by a host application, a fixed memory budget
// reserved at start-up, a real-time loop that must not enter the driver's
// allocator).  Its scratch is a fixed device global instead of a workspace
// argument.

namespace fa {
namespace {

// The FP32 dQ accumulator and D for fa_bwd_noalloc.  Every GPU that loads
// this library holds it until the process exits.  In host code this name is
// only a handle for cudaGetSymbolAddress, never a device address.
__device__ __align__(256) uint8_t g_bwd_scratch[FA_BWD_NOALLOC_SCRATCH_BYTES];

struct ScratchState {
  std::once_flag once;
  void* ptr = nullptr;   // device address of g_bwd_scratch on this device
};
ScratchState g_scratch[kMaxDevices];

// Looked up once per device, on the first fa_bwd_noalloc call made with that
// device current.  The lookup may load the module, so that first call must
// not happen inside a stream capture.
void* bwd_scratch() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  ScratchState* st = &g_scratch[dev];
  std::call_once(st->once, [st] {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_bwd_scratch) == cudaSuccess) st->ptr = ptr;
  });
  return st->ptr;
}

}  // namespace
}  // namespace fa

extern "C" int fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse,
                              const void* dout, void* dq, void* dk, void* dv, int B, int H, int N, int d,
                              int causal, float scale, void* stream) {
  if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv) return FA_ERR_NULL;
  const int rc = check_common(B, H, N, d, causal, scale);
  if (rc != FA_OK) return rc;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) || !aligned16(dq) ||
      !aligned16(dk) || !aligned16(dv))
    return FA_ERR_ALIGN;
  if (fa_bwd_workspace_size(B, H, N, d) > FA_BWD_NOALLOC_SCRATCH_BYTES) return FA_ERR_SCRATCH_LIMIT;
  FA_DEVICE_OR_RETURN(st);
  (void)st;
  void* scratch = bwd_scratch();
  if (!scratch) return FA_ERR_DEVICE;
  // fa_bwd's first launch zeroes the accumulator and rewrites D, so what the
  // previous call left in the array does not matter.
  return fa_bwd(q, k, v, o, lse, dout, dq, dk, dv, scratch, FA_BWD_NOALLOC_SCRATCH_BYTES, B, H, N, d, causal,
                scale, stream);
}
