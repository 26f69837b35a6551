// C ABI of the fused rotate + FP4 quantizer (declared in include/fp4q.h): plan objects,
// host-side validation, kernel selection and launch on the caller's stream.
#include <cuda_runtime.h>

#include <cstdio>
#include <cstring>
#include <mutex>
#include <new>
#include <unordered_map>

#include "fp4q_host.cuh"

using namespace fp4q;
using namespace fp4q::host;

namespace fp4q {
namespace host {

namespace {
thread_local char g_last_cuda_error[kLastErrorBytes] = "";
std::mutex g_ctx_mu;
// kernel, context, the dynamic shared memory occupancy is computed for, threads per CTA
struct InfoKey {
  const void* kernel;
  uint64_t ctx;
  int smem, threads;
  bool operator==(const InfoKey& o) const {
    return kernel == o.kernel && ctx == o.ctx && smem == o.smem && threads == o.threads;
  }
};
struct InfoKeyHash {
  size_t operator()(const InfoKey& k) const {
    uint64_t h = reinterpret_cast<uint64_t>(k.kernel) * 0x9E3779B97F4A7C15ull;
    h ^= k.ctx + 0x632BE59BD9B4E019ull + (h << 6) + (h >> 2);
    h ^= (static_cast<uint64_t>(static_cast<uint32_t>(k.smem)) << 20) ^ static_cast<uint64_t>(k.threads);
    return static_cast<size_t>(h);
  }
};
std::mutex g_info_mu;
std::unordered_map<InfoKey, KernelInfo, InfoKeyHash> g_info;
std::mutex g_encode_mu;
EncodeTiledFn g_encode = nullptr;
}  // namespace

char* last_error_buffer() { return g_last_cuda_error; }

fp4q_status cuda_fail(cudaError_t e, const char* what) {
  std::snprintf(last_error_buffer(), kLastErrorBytes, "%s: %s (%s)", what, cudaGetErrorString(e),
                cudaGetErrorName(e));
  return FP4Q_ERR_CUDA;
}

// Identity of the CUDA context current on this thread (0 when none is current yet).  Kernel
// attributes and occupancy belong to a context: after cudaDeviceReset, or under a context the
// caller made current through the driver API, the module is loaded afresh, so the cache below
// is keyed on this identity rather than on the device index.
fp4q_status current_context_id(uint64_t* out) {
  typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
  typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_ctx_mu);
    if (!get_current || !get_id) {
      void* f1 = nullptr;
      void* f2 = nullptr;
      cudaDriverEntryPointQueryResult q1, q2;
      cudaError_t e = cudaGetDriverEntryPoint("cuCtxGetCurrent", &f1, cudaEnableDefault, &q1);
      if (e == cudaSuccess) e = cudaGetDriverEntryPoint("cuCtxGetId", &f2, cudaEnableDefault, &q2);
      if (e != cudaSuccess) return cuda_fail(e, "cudaGetDriverEntryPoint(cuCtxGetCurrent / cuCtxGetId)");
      if (q1 != cudaDriverEntryPointSuccess || q2 != cudaDriverEntryPointSuccess || !f1 || !f2)
        return cuda_fail(cudaErrorNotSupported, "cuCtxGetCurrent / cuCtxGetId");
      get_current = reinterpret_cast<CtxGetCurrentFn>(f1);
      get_id = reinterpret_cast<CtxGetIdFn>(f2);
    }
  }
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS) return cuda_fail(cudaErrorDeviceUninitialized, "cuCtxGetCurrent");
  unsigned long long id = 0;
  if (ctx && get_id(ctx, &id) != CUDA_SUCCESS) return cuda_fail(cudaErrorDeviceUninitialized, "cuCtxGetId");
  *out = ctx ? static_cast<uint64_t>(id) + 1 : 0;
  return FP4Q_OK;
}

fp4q_status bound_context_id(uint64_t* out) {
  fp4q_status st = current_context_id(out);
  if (st != FP4Q_OK || *out != 0) return st;
  // nothing is current on this thread yet: bind the current device's primary context, as the
  // runtime's first call on this thread that needs a context would (it displaces nothing)
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaSetDevice(dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaSetDevice");
  return current_context_id(out);
}

fp4q_status kernel_info_impl(const void* kernel, int smem_bytes, int threads, KernelInfo* out, int max_smem_bytes) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  const int attr_smem = max_smem_bytes > smem_bytes ? max_smem_bytes : smem_bytes;
  uint64_t ctx = 0;
  fp4q_status st = bound_context_id(&ctx);
  if (st != FP4Q_OK) return st;
  const InfoKey key{kernel, ctx, smem_bytes, threads};
  std::lock_guard<std::mutex> lk(g_info_mu);
  auto it = g_info.find(key);
  if (it != g_info.end()) {
    *out = it->second;
    return FP4Q_OK;
  }
  KernelInfo ki;
  e = cudaDeviceGetAttribute(&ki.sm_count, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, attr_smem);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
  // all of the unified L1 / shared storage as shared memory: these kernels stage through it
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(carveout)");
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&ki.ctas_per_sm, kernel, threads, smem_bytes);
  if (e != cudaSuccess) return cuda_fail(e, "cudaOccupancyMaxActiveBlocksPerMultiprocessor");
  if (ki.ctas_per_sm < 1) ki.ctas_per_sm = 1;
  g_info[key] = ki;
  *out = ki;
  return FP4Q_OK;
}

fp4q_status encode_fn(EncodeTiledFn* out) {
  std::lock_guard<std::mutex> lk(g_encode_mu);
  if (!g_encode) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDriverEntryPoint(cuTensorMapEncodeTiled)");
    if (q != cudaDriverEntryPointSuccess || !fn) return cuda_fail(cudaErrorNotSupported, "cuTensorMapEncodeTiled");
    g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  }
  *out = g_encode;
  return FP4Q_OK;
}

}  // namespace host
}  // namespace fp4q

namespace {

constexpr uint32_t kPlanMagic = 0xF4F4A11Cu;

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

bool valid_plan(fp4q_plan p) { return p != nullptr && p->magic == kPlanMagic; }

// A plan's device memory (the partial maxima, the error pass's scratch) was allocated in the
// CUDA context current when the plan was made (the device's primary context, unless the
// caller made another one current), so every call that launches must be made with that
// context current: another device, or another context on the same device, cannot reach it.
// Checked before anything is launched.
fp4q_status check_device(fp4q_plan p, const char* who) {
  if (p->device < 0) return FP4Q_OK;   // made without a device: it owns no device memory
  uint64_t ctx = 0;
  fp4q_status st = bound_context_id(&ctx);
  if (st != FP4Q_OK) return st;
  if (ctx != p->context) {
    int dev = -1;
    (void)cudaGetDevice(&dev);
    std::snprintf(last_error_buffer(), kLastErrorBytes,
                  "%s: the plan belongs to a CUDA context on device %d, but another context (device %d) is current",
                  who, p->device, dev);
    return FP4Q_ERR_ARG;
  }
  return FP4Q_OK;
}

// Whether the tensor-core kernel serves this plan.  AUTO takes it for tensors of at least
// kMmaMinElems elements: below that its fixed start-up (TMEM allocation, H_b, filling a
// three-stage pipeline) costs more than the butterfly kernel's extra instructions.  MXFP4
// plans with channel signs and b = 128 go to the butterfly kernel from kSignedMxMmaMaxElems
// elements on: there the tensor-core kernel's pass that flips the signs in each landed stage
// holds it near 80 % of HBM bandwidth, where the butterfly, which flips them as it loads, runs
// at 84-87 %; below, the tensor core is the faster of the two (73-84 % against 65-80 %,
// measured from 4096 x 8192 to 32768 x 14336).
constexpr int64_t kMmaMinElems = int64_t(1) << 22;
constexpr int64_t kSignedMxMmaMaxElems = int64_t(3) << 26;
bool mma_capable(fp4q_plan p) { return p->block >= 16 && p->block >= p->group; }
// The tensor-core kernel addresses its tiles with 32-bit TMA coordinates (rows of one Hadamard
// block each); larger tensors go to the butterfly kernel.
constexpr int64_t kMmaMaxRows = (int64_t(1) << 31) - 1024;
bool use_mma(fp4q_plan p, int64_t n_elems) {
  if (!mma_capable(p) || n_elems / p->block >= kMmaMaxRows) return false;
  if (p->kernel == FP4Q_KERNEL_TENSOR_CORE) return true;
  if (p->signs && p->format == FP4Q_MXFP4 && p->block == 128 && n_elems >= kSignedMxMmaMaxElems) return false;
  return p->kernel == FP4Q_KERNEL_AUTO && n_elems >= kMmaMinElems;
}

// Number of CTAs the amax pass always launches (and of partial maxima a plan holds): one
// full wave of the larger of its two instances.
fp4q_status amax_grid(int b, int* n) {
  return with_block(b, [&]<int B>() -> fp4q_status {
    int a = 0, c = 0;
    fp4q_status st = amax_wave<AmaxCfg<B, 16>>(&a);
    if (st != FP4Q_OK) return st;
    st = amax_wave<AmaxCfg<B, 32>>(&c);
    if (st != FP4Q_OK) return st;
    *n = a > c ? a : c;
    return FP4Q_OK;
  });
}

// The amax pass runs on the tensor-core kernel where the plan's rotate + quantize calls would
// (b >= 16; AUTO from kMmaMinElems elements on): its 32 KB stages keep HBM busier than the
// butterfly kernel's 2 KB copies.  A plan held to the butterfly kernel keeps its amax pass
// there too, so that its maxima come from the same fp32 sums.
fp4q_status launch_amax(fp4q_plan p, const uint16_t* x, int64_t n_elems, int64_t K, cudaStream_t stream) {
  // (an empty tensor takes the butterfly kernel, whose fixed grid writes every slot)
  const bool tc = n_elems > 0 && p->block >= 16 && n_elems / p->block < kMmaMaxRows &&
                  p->kernel != FP4Q_KERNEL_BUTTERFLY && (p->kernel == FP4Q_KERNEL_TENSOR_CORE || n_elems >= kMmaMinElems);
  if (tc) {
    return with_block(p->block, [&]<int B>() -> fp4q_status {
      if constexpr (B >= 16)
        return launch_mma_amax<MmaConfig<kNV, B, kRuleNvStatic, false, false, true>>(
            x, n_elems, p->partials, p->n_partials, ChannelSigns{p->signs, 1, 0}, stream, K);
      return FP4Q_ERR_UNSUPPORTED;
    });
  }
  return with_block(p->block, [&]<int B>() -> fp4q_status {
    if (n_elems % AmaxCfg<B, 32>::kE == 0)
      return launch_amax_cfg<AmaxCfg<B, 32>>(x, n_elems, p->partials, p->n_partials,
                                             channel_signs<AmaxCfg<B, 32>>(p->signs, p->signs_K), stream, true);
    return launch_amax_cfg<AmaxCfg<B, 16>>(x, n_elems, p->partials, p->n_partials,
                                           channel_signs<AmaxCfg<B, 16>>(p->signs, p->signs_K), stream, true);
  });
}

fp4q_status check_shape(fp4q_plan p, int64_t M, int64_t K) {
  if (M < 0 || K < 0) return FP4Q_ERR_SHAPE;
  if (p->signs && K != p->signs_K) return FP4Q_ERR_SHAPE;   // the signs are for rows of signs_K
  if (K % p->unit != 0) return FP4Q_ERR_SHAPE;  // unit = lcm(group, block) for powers of two
  if (M > 0 && K > 0 && M > (int64_t(1) << 40) / K) return FP4Q_ERR_SHAPE;
  return FP4Q_OK;
}

fp4q_status rotate_quantize_impl(fp4q_plan p, const void* x, int64_t M, int64_t K, void* codes, void* scales,
                                 float* tensor_scale, float* y_out, bool dump, void* stream, void* macro = nullptr) {
  if (!valid_plan(p)) return FP4Q_ERR_ARG;
  // an MBS plan also stores macro-scale bytes: only fp4q_rotate_quantize_mbs (macro != null) serves it
  if ((p->format == FP4Q_MXFP4_MBS) != (macro != nullptr)) return FP4Q_ERR_UNSUPPORTED;
  fp4q_status st = check_device(p, "fp4q_rotate_quantize");
  if (st != FP4Q_OK) return st;
  st = check_shape(p, M, K);
  if (st != FP4Q_OK) return st;
  if (M * K == 0) return FP4Q_OK;
  if (!x || !codes || !scales || (dump && !y_out)) return FP4Q_ERR_ARG;
  if (p->format == FP4Q_NVFP4 && !tensor_scale) return FP4Q_ERR_ARG;
  if (!aligned(x, 16) || !aligned(codes, 16) || !aligned(scales, 16) || (dump && !aligned(y_out, 16)) ||
      (tensor_scale && !aligned(tensor_scale, 4)))
    return FP4Q_ERR_ALIGN;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  RQArgs a;
  const int64_t n = M * K;
  a.x = static_cast<const uint16_t*>(x);
  a.n_units = 0;  // set per instance from its unit size
  a.codes = static_cast<uint8_t*>(codes);
  a.scales = static_cast<uint8_t*>(scales);
  a.tensor_scale = tensor_scale;
  a.partials = p->partials;
  a.n_partials = p->n_partials;
  a.y_dump = y_out;
  a.signs = ChannelSigns{p->signs, 1, 0};
  a.macro = static_cast<uint8_t*>(macro);
  if (p->format == FP4Q_NVFP4 && p->rule == FP4Q_SCALE_NV_DYNAMIC) {
    st = launch_amax(p, a.x, n, K, s);
    if (st != FP4Q_OK) return st;
  }
  if (use_mma(p, n)) {
    return with_block(p->block, [&]<int B>() -> fp4q_status {
      if constexpr (B >= 16) {
        if (p->format == FP4Q_MXFP4_MBS) {
          // the MBS entry has no dump form (it was refused above when macro is null)
          if constexpr (B >= 32) {
            switch (p->rule) {
              case FP4Q_SCALE_FLOOR_OCP: return launch_mma<MmaConfig<kMBS, B, kRuleFloor, false>>(a.x, n, a, s, K);
              case FP4Q_SCALE_CEIL_NOCLIP: return launch_mma<MmaConfig<kMBS, B, kRuleCeil, false>>(a.x, n, a, s, K);
              case FP4Q_SCALE_OAS: return launch_mma<MmaConfig<kMBS, B, kRuleOas, false>>(a.x, n, a, s, K);
              default: return FP4Q_ERR_UNSUPPORTED;
            }
          }
          return FP4Q_ERR_UNSUPPORTED;
        }
        if (p->format == FP4Q_MXFP4) {
          if constexpr (B >= 32) {
            switch (p->rule) {
              case FP4Q_SCALE_FLOOR_OCP:
                return dump ? launch_mma<MmaConfig<kMX, B, kRuleFloor, true>>(a.x, n, a, s, K)
                            : launch_mma<MmaConfig<kMX, B, kRuleFloor, false>>(a.x, n, a, s, K);
              case FP4Q_SCALE_CEIL_NOCLIP:
                return dump ? launch_mma<MmaConfig<kMX, B, kRuleCeil, true>>(a.x, n, a, s, K)
                            : launch_mma<MmaConfig<kMX, B, kRuleCeil, false>>(a.x, n, a, s, K);
              case FP4Q_SCALE_OAS:
                return dump ? launch_mma<MmaConfig<kMX, B, kRuleOas, true>>(a.x, n, a, s, K)
                            : launch_mma<MmaConfig<kMX, B, kRuleOas, false>>(a.x, n, a, s, K);
              default: return FP4Q_ERR_UNSUPPORTED;
            }
          }
          return FP4Q_ERR_UNSUPPORTED;
        }
        if (p->rule == FP4Q_SCALE_NV_DYNAMIC)
          return dump ? launch_mma<MmaConfig<kNV, B, kRuleNvDynamic, true>>(a.x, n, a, s, K)
                      : launch_mma<MmaConfig<kNV, B, kRuleNvDynamic, false>>(a.x, n, a, s, K);
        return dump ? launch_mma<MmaConfig<kNV, B, kRuleNvStatic, true>>(a.x, n, a, s, K)
                    : launch_mma<MmaConfig<kNV, B, kRuleNvStatic, false>>(a.x, n, a, s, K);
      }
      return FP4Q_ERR_UNSUPPORTED;
    });
  }
  return with_block(p->block, [&]<int B>() -> fp4q_status {
    if (p->format == FP4Q_MXFP4_MBS) {
      switch (p->rule) {
        case FP4Q_SCALE_FLOOR_OCP: return launch_rq<RQConfig<kMBS, B, kRuleFloor, false, 128>>(a, n, s, K);
        case FP4Q_SCALE_CEIL_NOCLIP: return launch_rq<RQConfig<kMBS, B, kRuleCeil, false, 128>>(a, n, s, K);
        case FP4Q_SCALE_OAS: return launch_rq<RQConfig<kMBS, B, kRuleOas, false, 128>>(a, n, s, K);
        default: return FP4Q_ERR_UNSUPPORTED;
      }
    }
    if (p->format == FP4Q_MXFP4) {
      switch (p->rule) {
        case FP4Q_SCALE_FLOOR_OCP:
          return dump ? launch_rq<RQConfig<kMX, B, kRuleFloor, true>>(a, n, s, K)
                      : launch_rq<RQConfig<kMX, B, kRuleFloor, false>>(a, n, s, K);
        case FP4Q_SCALE_CEIL_NOCLIP:
          return dump ? launch_rq<RQConfig<kMX, B, kRuleCeil, true>>(a, n, s, K)
                      : launch_rq<RQConfig<kMX, B, kRuleCeil, false>>(a, n, s, K);
        case FP4Q_SCALE_OAS:
          return dump ? launch_rq<RQConfig<kMX, B, kRuleOas, true>>(a, n, s, K)
                      : launch_rq<RQConfig<kMX, B, kRuleOas, false>>(a, n, s, K);
        default: return FP4Q_ERR_UNSUPPORTED;
      }
    }
    // NVFP4: 32-element units when the element count allows, else 16
    const bool u32 = n % 32 == 0;
    if (p->rule == FP4Q_SCALE_NV_DYNAMIC) {
      if (u32)
        return dump ? launch_rq<RQConfig<kNV, B, kRuleNvDynamic, true, 32>>(a, n, s, K)
                    : launch_rq<RQConfig<kNV, B, kRuleNvDynamic, false, 32>>(a, n, s, K);
      return dump ? launch_rq<RQConfig<kNV, B, kRuleNvDynamic, true, 16>>(a, n, s, K)
                  : launch_rq<RQConfig<kNV, B, kRuleNvDynamic, false, 16>>(a, n, s, K);
    }
    if (u32)
      return dump ? launch_rq<RQConfig<kNV, B, kRuleNvStatic, true, 32>>(a, n, s, K)
                  : launch_rq<RQConfig<kNV, B, kRuleNvStatic, false, 32>>(a, n, s, K);
    return dump ? launch_rq<RQConfig<kNV, B, kRuleNvStatic, true, 16>>(a, n, s, K)
                : launch_rq<RQConfig<kNV, B, kRuleNvStatic, false, 16>>(a, n, s, K);
  });
}

// ---- quantization error energies (butterfly kernel for every block size)

// Call f.template operator()<Cfg>() for the butterfly configuration of (format, block, rule);
// NVFP4 takes 32-element units when the element count allows (u32), else 16.
template <class F>
fp4q_status with_rq_cfg(int format, int block, int rule, bool u32, F&& f) {
  return with_block(block, [&]<int B>() -> fp4q_status {
    if (format == FP4Q_MXFP4_MBS) {
      switch (rule) {
        case FP4Q_SCALE_FLOOR_OCP: return f.template operator()<RQConfig<kMBS, B, kRuleFloor, false, 128>>();
        case FP4Q_SCALE_CEIL_NOCLIP: return f.template operator()<RQConfig<kMBS, B, kRuleCeil, false, 128>>();
        case FP4Q_SCALE_OAS: return f.template operator()<RQConfig<kMBS, B, kRuleOas, false, 128>>();
        default: return FP4Q_ERR_UNSUPPORTED;
      }
    }
    if (format == FP4Q_MXFP4) {
      switch (rule) {
        case FP4Q_SCALE_FLOOR_OCP: return f.template operator()<RQConfig<kMX, B, kRuleFloor, false>>();
        case FP4Q_SCALE_CEIL_NOCLIP: return f.template operator()<RQConfig<kMX, B, kRuleCeil, false>>();
        case FP4Q_SCALE_OAS: return f.template operator()<RQConfig<kMX, B, kRuleOas, false>>();
        default: return FP4Q_ERR_UNSUPPORTED;
      }
    }
    if (rule == FP4Q_SCALE_NV_DYNAMIC)
      return u32 ? f.template operator()<RQConfig<kNV, B, kRuleNvDynamic, false, 32>>()
                 : f.template operator()<RQConfig<kNV, B, kRuleNvDynamic, false, 16>>();
    return u32 ? f.template operator()<RQConfig<kNV, B, kRuleNvStatic, false, 32>>()
               : f.template operator()<RQConfig<kNV, B, kRuleNvStatic, false, 16>>();
  });
}

// CTAs of one full wave of the error kernel for the plan, over both unit sizes.
fp4q_status qe_grid(int format, int block, int rule, int* n) {
  *n = 0;
  for (int u32 = 0; u32 < 2; ++u32) {
    fp4q_status st = with_rq_cfg(format, block, rule, u32 != 0, [&]<class Cfg>() -> fp4q_status {
      int w = 0;
      fp4q_status r = qe_wave<Cfg>(&w);
      if (r == FP4Q_OK && w > *n) *n = w;
      return r;
    });
    if (st != FP4Q_OK) return st;
  }
  // the tensor-core error pass: at most two persistent CTAs per SM
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
  if (2 * sms > *n) *n = 2 * sms;
  return FP4Q_OK;
}

// ---- no-allocation NVFP4 dynamic path: partial maxima in a fixed device array

// Device address of the no-allocation scratch in the context current now.  Looked up on every
// call (a host-side lookup): an address kept from an earlier call would be stale after
// cudaDeviceReset, or under another context the caller made current.
fp4q_status noalloc_scratch(float** out) {
  float* ptr = nullptr;
  fp4q_status st = noalloc_partials_symbol(&ptr);
  if (st != FP4Q_OK) return st;
  *out = ptr;
  return FP4Q_OK;
}

}  // namespace

extern "C" {

fp4q_status fp4q_rotate_quantize_nvfp4_dynamic_noalloc(const void* x_bf16, int64_t M, int64_t K, int hadamard_block,
                                                       void* codes_out, void* scales_out, float* tensor_scale_out,
                                                       void* stream) {
  if (hadamard_block < 1 || hadamard_block > 128 || (hadamard_block & (hadamard_block - 1)) != 0)
    return FP4Q_ERR_UNSUPPORTED;
  const int64_t unit = hadamard_block > 16 ? hadamard_block : 16;
  if (M < 0 || K < 0 || K % unit != 0) return FP4Q_ERR_SHAPE;
  if (M > 0 && K > 0 && M > (int64_t(1) << 40) / K) return FP4Q_ERR_SHAPE;
  if (!tensor_scale_out) return FP4Q_ERR_ARG;
  if (M * K == 0) return FP4Q_OK;
  if (!x_bf16 || !codes_out || !scales_out) return FP4Q_ERR_ARG;
  if (!aligned(x_bf16, 16) || !aligned(codes_out, 16) || !aligned(scales_out, 16) || !aligned(tensor_scale_out, 4))
    return FP4Q_ERR_ALIGN;
  float* partials = nullptr;
  fp4q_status st = noalloc_scratch(&partials);
  if (st != FP4Q_OK) return st;
  int n_partials = 0;
  st = amax_grid(hadamard_block, &n_partials);
  if (st != FP4Q_OK) return st;
  if (n_partials > kNoAllocMaxPartials) {
    std::snprintf(last_error_buffer(), kLastErrorBytes,
                  "fp4q_rotate_quantize_nvfp4_dynamic_noalloc: the amax pass needs %d partial maxima, "
                  "the fixed scratch holds %d",
                  n_partials, kNoAllocMaxPartials);
    return FP4Q_ERR_UNSUPPORTED;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t n = M * K;
  const uint16_t* x = static_cast<const uint16_t*>(x_bf16);
  RQArgs a;
  a.x = x;
  a.n_units = 0;
  a.codes = static_cast<uint8_t*>(codes_out);
  a.scales = static_cast<uint8_t*>(scales_out);
  a.tensor_scale = tensor_scale_out;
  a.partials = partials;
  a.n_partials = n_partials;
  a.y_dump = nullptr;
  a.signs = ChannelSigns{nullptr, 1, 0};
  a.macro = nullptr;
  return with_block(hadamard_block, [&]<int B>() -> fp4q_status {
    if (n % 32 == 0) {
      fp4q_status r = launch_amax_cfg<AmaxCfg<B, 32>>(x, n, partials, n_partials, ChannelSigns{nullptr, 1, 0}, s, false);
      if (r != FP4Q_OK) return r;
      return launch_rq<RQConfig<kNV, B, kRuleNvDynamic, false, 32>>(a, n, s);
    }
    fp4q_status r = launch_amax_cfg<AmaxCfg<B, 16>>(x, n, partials, n_partials, ChannelSigns{nullptr, 1, 0}, s, false);
    if (r != FP4Q_OK) return r;
    return launch_rq<RQConfig<kNV, B, kRuleNvDynamic, false, 16>>(a, n, s);
  });
}

fp4q_status fp4q_plan_create(fp4q_plan* out, int format, int group, int hadamard_block, int scale_rule) {
  if (!out) return FP4Q_ERR_ARG;
  *out = nullptr;
  if (format == FP4Q_MXFP4 || format == FP4Q_MXFP4_MBS) {
    if (group != 32) return FP4Q_ERR_UNSUPPORTED;
    if (scale_rule != FP4Q_SCALE_FLOOR_OCP && scale_rule != FP4Q_SCALE_CEIL_NOCLIP && scale_rule != FP4Q_SCALE_OAS)
      return FP4Q_ERR_UNSUPPORTED;
  } else if (format == FP4Q_NVFP4) {
    if (group != 16) return FP4Q_ERR_UNSUPPORTED;
    if (scale_rule != FP4Q_SCALE_NV_STATIC && scale_rule != FP4Q_SCALE_NV_DYNAMIC) return FP4Q_ERR_UNSUPPORTED;
  } else {
    return FP4Q_ERR_UNSUPPORTED;
  }
  if (hadamard_block < 1 || hadamard_block > 128 || (hadamard_block & (hadamard_block - 1)) != 0)
    return FP4Q_ERR_UNSUPPORTED;
  fp4q_plan p = new (std::nothrow) fp4q_plan_s();
  if (!p) return FP4Q_ERR_ARG;
  p->magic = kPlanMagic;
  p->format = format;
  p->group = group;
  p->block = hadamard_block;
  p->rule = scale_rule;
  p->unit = group > hadamard_block ? group : hadamard_block;
  if (format == FP4Q_MXFP4_MBS) p->unit = 128;   // one macro block per unit (b <= 128)
  p->device = -1;
  p->context = 0;
  p->partials = nullptr;
  p->n_partials = 0;
  p->kernel = FP4Q_KERNEL_AUTO;
  p->err_partials = nullptr;
  p->n_err_partials = 0;
  p->signs = nullptr;
  p->signs_K = 0;
  fp4q_status st = FP4Q_OK;
  if (format == FP4Q_NVFP4) {
    cudaError_t e = cudaGetDevice(&p->device);
    st = e == cudaSuccess ? amax_grid(hadamard_block, &p->n_partials) : cuda_fail(e, "cudaGetDevice");
    if (st == FP4Q_OK) {
      e = cudaMalloc(&p->partials, sizeof(float) * static_cast<size_t>(p->n_partials));
      if (e != cudaSuccess) st = cuda_fail(e, "cudaMalloc partials");
    }
  } else {
    // an MX plan needs a device only for fp4q_quant_error's scratch: without one it is still made
    int ndev = 0;
    if (cudaGetDeviceCount(&ndev) != cudaSuccess || ndev == 0) {
      (void)cudaGetLastError();
      *out = p;
      return FP4Q_OK;
    }
    cudaError_t e = cudaGetDevice(&p->device);
    if (e != cudaSuccess) st = cuda_fail(e, "cudaGetDevice");
  }
  if (st == FP4Q_OK) st = qe_grid(format, hadamard_block, scale_rule, &p->n_err_partials);
  if (st == FP4Q_OK) {
    // the partial pairs, then the ticket counter (zeroed once; each call's last CTA re-zeroes it)
    const size_t bytes = (2 * static_cast<size_t>(p->n_err_partials) + 1) * sizeof(double);
    cudaError_t e = cudaMalloc(&p->err_partials, bytes);
    if (e == cudaSuccess) e = cudaMemset(p->err_partials, 0, bytes);
    if (e != cudaSuccess) st = cuda_fail(e, "cudaMalloc error partials");
  }
  if (st == FP4Q_OK) st = bound_context_id(&p->context);   // the context the allocations were made in
  if (st != FP4Q_OK) {
    if (p->partials) cudaFree(p->partials);
    if (p->err_partials) cudaFree(p->err_partials);
    p->magic = 0;
    delete p;
    return st;
  }
  *out = p;
  return FP4Q_OK;
}

fp4q_status fp4q_plan_set_kernel(fp4q_plan plan, int kernel) {
  if (!valid_plan(plan)) return FP4Q_ERR_ARG;
  if (kernel != FP4Q_KERNEL_AUTO && kernel != FP4Q_KERNEL_BUTTERFLY && kernel != FP4Q_KERNEL_TENSOR_CORE)
    return FP4Q_ERR_ARG;
  if (kernel == FP4Q_KERNEL_TENSOR_CORE && !mma_capable(plan)) return FP4Q_ERR_UNSUPPORTED;
  plan->kernel = kernel;
  return FP4Q_OK;
}

fp4q_status fp4q_plan_set_signs(fp4q_plan plan, const uint32_t* signs, int64_t K) {
  if (!valid_plan(plan)) return FP4Q_ERR_ARG;
  if (!signs) {
    plan->signs = nullptr;
    plan->signs_K = 0;
    return FP4Q_OK;
  }
  if (K <= 0 || K % plan->unit != 0 || K > (int64_t(1) << 34)) return FP4Q_ERR_SHAPE;
  if (!aligned(signs, 4)) return FP4Q_ERR_ALIGN;
  plan->signs = signs;
  plan->signs_K = K;
  return FP4Q_OK;
}

fp4q_status fp4q_plan_destroy(fp4q_plan plan) {
  if (!plan) return FP4Q_OK;
  if (!valid_plan(plan)) return FP4Q_ERR_ARG;
  fp4q_status st = FP4Q_OK;
  if (plan->partials) {
    cudaError_t e = cudaFree(plan->partials);
    if (e != cudaSuccess) st = cuda_fail(e, "cudaFree partials");
  }
  if (plan->err_partials) {
    cudaError_t e = cudaFree(plan->err_partials);
    if (e != cudaSuccess) st = cuda_fail(e, "cudaFree error partials");
  }
  plan->magic = 0;
  delete plan;
  return st;
}

fp4q_status fp4q_rotate_quantize(fp4q_plan plan, const void* x_bf16, int64_t M, int64_t K, void* codes_out,
                                 void* scales_out, float* tensor_scale, void* stream) {
  return rotate_quantize_impl(plan, x_bf16, M, K, codes_out, scales_out, tensor_scale, nullptr, false, stream);
}

fp4q_status fp4q_rotate_quantize_mbs(fp4q_plan plan, const void* x_bf16, int64_t M, int64_t K, void* codes_out,
                                     void* scales_out, void* macro_out, void* stream) {
  if (!valid_plan(plan)) return FP4Q_ERR_ARG;
  if (plan->format != FP4Q_MXFP4_MBS) return FP4Q_ERR_UNSUPPORTED;
  if (!macro_out) return M * K == 0 && M >= 0 && K >= 0 ? FP4Q_OK : FP4Q_ERR_ARG;
  return rotate_quantize_impl(plan, x_bf16, M, K, codes_out, scales_out, nullptr, nullptr, false, stream, macro_out);
}

fp4q_status fp4q_rotate_quantize_dump(fp4q_plan plan, const void* x_bf16, int64_t M, int64_t K, void* codes_out,
                                      void* scales_out, float* tensor_scale, float* y_out, void* stream) {
  return rotate_quantize_impl(plan, x_bf16, M, K, codes_out, scales_out, tensor_scale, y_out, true, stream);
}

fp4q_status fp4q_amax(fp4q_plan plan, const void* x_bf16, int64_t M, int64_t K, float* tensor_scale_out,
                      void* stream) {
  if (!valid_plan(plan)) return FP4Q_ERR_ARG;
  if (plan->format != FP4Q_NVFP4) return FP4Q_ERR_UNSUPPORTED;
  fp4q_status st = check_device(plan, "fp4q_amax");
  if (st != FP4Q_OK) return st;
  st = check_shape(plan, M, K);
  if (st != FP4Q_OK) return st;
  if (!tensor_scale_out) return FP4Q_ERR_ARG;
  if (M * K > 0 && !x_bf16) return FP4Q_ERR_ARG;
  if ((x_bf16 && !aligned(x_bf16, 16)) || !aligned(tensor_scale_out, 4)) return FP4Q_ERR_ALIGN;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  st = launch_amax(plan, static_cast<const uint16_t*>(x_bf16), M * K, K, s);
  if (st != FP4Q_OK) return st;
  return launch_tensor_scale_finalize(plan->partials, plan->n_partials, tensor_scale_out, s);
}

fp4q_status fp4q_quant_error(fp4q_plan plan, const void* x_bf16, int64_t M, int64_t K, float* tensor_scale,
                             double* out, void* stream) {
  if (!valid_plan(plan)) return FP4Q_ERR_ARG;
  fp4q_status st = check_device(plan, "fp4q_quant_error");
  if (st != FP4Q_OK) return st;
  st = check_shape(plan, M, K);
  if (st != FP4Q_OK) return st;
  if (!out) return FP4Q_ERR_ARG;
  if (plan->format == FP4Q_NVFP4 && !tensor_scale) return FP4Q_ERR_ARG;
  if (M * K > 0 && !x_bf16) return FP4Q_ERR_ARG;
  if ((x_bf16 && !aligned(x_bf16, 16)) || !aligned(out, 8) || (tensor_scale && !aligned(tensor_scale, 4)))
    return FP4Q_ERR_ALIGN;
  if (!plan->err_partials) {
    std::snprintf(last_error_buffer(), kLastErrorBytes,
                  "fp4q_quant_error: the plan was made without a CUDA device, so it holds no scratch");
    return FP4Q_ERR_UNSUPPORTED;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t n = M * K;
  if (n == 0) {
    return launch_quant_error_empty(plan->err_partials, out, s);
  }
  QEArgs a;
  a.x = static_cast<const uint16_t*>(x_bf16);
  a.n_units = 0;
  a.tensor_scale = tensor_scale;
  a.partials = plan->partials;
  a.n_partials = plan->n_partials;
  a.out_partials = plan->err_partials;
  a.ticket = reinterpret_cast<unsigned int*>(plan->err_partials + 2 * static_cast<int64_t>(plan->n_err_partials));
  a.out = out;
  if (plan->format == FP4Q_NVFP4 && plan->rule == FP4Q_SCALE_NV_DYNAMIC) {
    st = launch_amax(plan, a.x, n, K, s);
    if (st != FP4Q_OK) return st;
  }
  if (use_mma(plan, n)) {
    // the kernel fp4q_rotate_quantize picks for this plan and size, so the same codes
    a.signs = ChannelSigns{plan->signs, 1, 0};
    const int slots = plan->n_err_partials;
    return with_block(plan->block, [&]<int B>() -> fp4q_status {
      if constexpr (B >= 16) {
        if (plan->format == FP4Q_MXFP4_MBS) {
          if constexpr (B >= 32) {
            switch (plan->rule) {
              case FP4Q_SCALE_FLOOR_OCP:
                return launch_mma_qe<MmaConfig<kMBS, B, kRuleFloor, false, true>>(a, n, s, K, slots);
              case FP4Q_SCALE_CEIL_NOCLIP:
                return launch_mma_qe<MmaConfig<kMBS, B, kRuleCeil, false, true>>(a, n, s, K, slots);
              case FP4Q_SCALE_OAS:
                return launch_mma_qe<MmaConfig<kMBS, B, kRuleOas, false, true>>(a, n, s, K, slots);
              default: return FP4Q_ERR_UNSUPPORTED;
            }
          }
          return FP4Q_ERR_UNSUPPORTED;
        }
        if (plan->format == FP4Q_MXFP4) {
          if constexpr (B >= 32) {
            switch (plan->rule) {
              case FP4Q_SCALE_FLOOR_OCP:
                return launch_mma_qe<MmaConfig<kMX, B, kRuleFloor, false, true>>(a, n, s, K, slots);
              case FP4Q_SCALE_CEIL_NOCLIP:
                return launch_mma_qe<MmaConfig<kMX, B, kRuleCeil, false, true>>(a, n, s, K, slots);
              case FP4Q_SCALE_OAS:
                return launch_mma_qe<MmaConfig<kMX, B, kRuleOas, false, true>>(a, n, s, K, slots);
              default: return FP4Q_ERR_UNSUPPORTED;
            }
          }
          return FP4Q_ERR_UNSUPPORTED;
        }
        if (plan->rule == FP4Q_SCALE_NV_DYNAMIC)
          return launch_mma_qe<MmaConfig<kNV, B, kRuleNvDynamic, false, true>>(a, n, s, K, slots);
        return launch_mma_qe<MmaConfig<kNV, B, kRuleNvStatic, false, true>>(a, n, s, K, slots);
      }
      return FP4Q_ERR_UNSUPPORTED;
    });
  }
  return with_rq_cfg(plan->format, plan->block, plan->rule, n % 32 == 0,
                     [&]<class Cfg>() -> fp4q_status { return launch_qe<Cfg>(plan, a, n, out, s); });
}

namespace {
fp4q_status dequantize_impl(fp4q_plan plan, const void* codes, const void* scales, const void* macro,
                            const float* tensor_scale, int64_t M, int64_t K, int unrotate, float* out_f32,
                            void* stream) {
  fp4q_status st = check_device(plan, "fp4q_dequantize");
  if (st != FP4Q_OK) return st;
  st = check_shape(plan, M, K);
  if (st != FP4Q_OK) return st;
  if (M * K == 0) return FP4Q_OK;
  if (!codes || !scales || !out_f32 || (plan->format == FP4Q_NVFP4 && !tensor_scale)) return FP4Q_ERR_ARG;
  if (!aligned(codes, 16) || !aligned(scales, 16) || !aligned(out_f32, 16) ||
      (tensor_scale && !aligned(tensor_scale, 4)))
    return FP4Q_ERR_ALIGN;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t n_units = (M * K) / plan->unit;
  const uint8_t* c = static_cast<const uint8_t*>(codes);
  const uint8_t* sc = static_cast<const uint8_t*>(scales);
  st = with_block(plan->block, [&]<int B>() -> fp4q_status {
    // the dequantize kernel's unit is the plan's, E = max(g, b)
    const ChannelSigns dsg = plan->signs ? ChannelSigns{plan->signs, static_cast<int>(plan->signs_K / plan->unit), 0}
                                         : ChannelSigns{nullptr, 1, 0};
    const uint8_t* mc = static_cast<const uint8_t*>(macro);
    if (plan->format == FP4Q_MXFP4_MBS) {
      if (unrotate) return launch_dequantize<kMBS, B, true>(c, sc, tensor_scale, n_units, out_f32, dsg, mc, s);
      else return launch_dequantize<kMBS, B, false>(c, sc, tensor_scale, n_units, out_f32, dsg, mc, s);
    } else if (plan->format == FP4Q_MXFP4) {
      if (unrotate) return launch_dequantize<kMX, B, true>(c, sc, tensor_scale, n_units, out_f32, dsg, mc, s);
      else return launch_dequantize<kMX, B, false>(c, sc, tensor_scale, n_units, out_f32, dsg, mc, s);
    } else {
      if (unrotate) return launch_dequantize<kNV, B, true>(c, sc, tensor_scale, n_units, out_f32, dsg, mc, s);
      else return launch_dequantize<kNV, B, false>(c, sc, tensor_scale, n_units, out_f32, dsg, mc, s);
    }
  });
  return st;
}
}  // namespace

fp4q_status fp4q_dequantize(fp4q_plan plan, const void* codes, const void* scales, const float* tensor_scale,
                            int64_t M, int64_t K, int unrotate, float* out_f32, void* stream) {
  if (!valid_plan(plan)) return FP4Q_ERR_ARG;
  if (plan->format == FP4Q_MXFP4_MBS) return FP4Q_ERR_UNSUPPORTED;   // needs the macro scales
  return dequantize_impl(plan, codes, scales, nullptr, tensor_scale, M, K, unrotate, out_f32, stream);
}

fp4q_status fp4q_dequantize_mbs(fp4q_plan plan, const void* codes, const void* scales, const void* macro, int64_t M,
                                int64_t K, int unrotate, float* out_f32, void* stream) {
  if (!valid_plan(plan)) return FP4Q_ERR_ARG;
  if (plan->format != FP4Q_MXFP4_MBS) return FP4Q_ERR_UNSUPPORTED;
  if (M * K > 0 && !macro) return FP4Q_ERR_ARG;
  return dequantize_impl(plan, codes, scales, macro, nullptr, M, K, unrotate, out_f32, stream);
}

fp4q_status fp4q_gemm(int format, const void* a_codes, const void* a_scales, const float* a_tensor_scale,
                      const void* b_codes, const void* b_scales, const float* b_tensor_scale, int64_t M, int64_t N,
                      int64_t K, void* d_bf16, void* stream) {
  if (format != FP4Q_MXFP4 && format != FP4Q_NVFP4) return FP4Q_ERR_UNSUPPORTED;
  if (M < 0 || N < 0 || K < 0 || N % 32 != 0 || K % 256 != 0) return FP4Q_ERR_SHAPE;
  if (M > (int64_t(1) << 31) || N > (int64_t(1) << 31) || (K > 0 && (M > (int64_t(1) << 40) / K ||
                                                                        N > (int64_t(1) << 40) / K)))
    return FP4Q_ERR_SHAPE;
  if (M == 0 || N == 0) return FP4Q_OK;
  if (K == 0) return FP4Q_ERR_SHAPE;   // an empty reduction: no MMA would write the accumulator
  if (!a_codes || !a_scales || !b_codes || !b_scales || !d_bf16) return FP4Q_ERR_ARG;
  if (format == FP4Q_NVFP4 && (!a_tensor_scale || !b_tensor_scale)) return FP4Q_ERR_ARG;
  if (!aligned(a_codes, 16) || !aligned(a_scales, 16) || !aligned(b_codes, 16) || !aligned(b_scales, 16) ||
      !aligned(d_bf16, 16) || (a_tensor_scale && !aligned(a_tensor_scale, 4)) ||
      (b_tensor_scale && !aligned(b_tensor_scale, 4)))
    return FP4Q_ERR_ALIGN;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const auto* ac = static_cast<const uint8_t*>(a_codes);
  const auto* as = static_cast<const uint8_t*>(a_scales);
  const auto* bc = static_cast<const uint8_t*>(b_codes);
  const auto* bs = static_cast<const uint8_t*>(b_scales);
  auto* d = static_cast<uint16_t*>(d_bf16);
  if (format == FP4Q_MXFP4) return launch_gemm<kMX>(ac, as, a_tensor_scale, bc, bs, b_tensor_scale, M, N, K, d, s);
  return launch_gemm<kNV>(ac, as, a_tensor_scale, bc, bs, b_tensor_scale, M, N, K, d, s);
}

fp4q_status fp4q_selftest_wait_timeout(void* stream) {
  return launch_wait_timeout_selftest(static_cast<cudaStream_t>(stream));
}

fp4q_status fp4q_device_status(void) {
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
  unsigned int v = 0;
  for (fp4q_status (*reader)(unsigned int*) : {status_rq_mx, status_rq_nv, status_mbs, status_qe, status_mma,
                                               status_mma_qe, status_dequant, status_gemm}) {
    fp4q_status st = reader(&v);
    if (st != FP4Q_OK) return st;
  }
  return (v & kStatusTimeout) ? FP4Q_ERR_TIMEOUT : FP4Q_OK;
}

const char* fp4q_status_string(fp4q_status status) {
  switch (status) {
    case FP4Q_OK: return "ok";
    case FP4Q_ERR_ARG: return "invalid argument";
    case FP4Q_ERR_SHAPE: return "invalid shape (K must be a multiple of max(group, hadamard_block))";
    case FP4Q_ERR_ALIGN: return "pointer not aligned (16 bytes for arrays, 4 for the tensor scale)";
    case FP4Q_ERR_UNSUPPORTED: return "unsupported format / group / block / rule";
    case FP4Q_ERR_CUDA: return "CUDA error";
    case FP4Q_ERR_TIMEOUT: return "a bounded wait inside a kernel ran out";
  }
  return "unknown status";
}

const char* fp4q_last_cuda_error(void) { return last_error_buffer(); }

int fp4q_version(void) { return 100; }

}  // extern "C"
