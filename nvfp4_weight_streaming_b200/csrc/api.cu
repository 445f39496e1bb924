// api.cu -- the C ABI declared in include/nvfp4_linear.h.
//
// Argument checking, plan construction (variant and split choice), and the
// launches. The library allocates no device memory; the caller passes every
// buffer, and PyTorch (or any other allocator) owns them.
#include "nvfp4_linear.h"
#include "kernels.h"

#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>
#include <cstdlib>
#include <cmath>
#include <mutex>
#include <new>

// Fixed split-K scratch behind nvfp4_linear_run_static: one copy per device
// (module globals are per device), shared by every call on that device.
static __device__ __align__(256) unsigned char g_static_scratch[NVFP4_STATIC_SCRATCH_BYTES];

namespace {
// TMA descriptors of one weight set, keyed by its two device pointers.
struct MapEntry {
  const void* wp = nullptr;
  const void* ws = nullptr;
  CUtensorMap mw, ms;
};
constexpr int kMapCache = 16;
}  // namespace

struct nvfp4_plan_s {
  int M, N, K, device;
  unsigned flags;
  int variant;
  int epi;        // fused epilogue: 0 none, 1 SwiGLU, 2 argmax (MMA variant only)
  int fmt;        // weight format: 0 NVFP4, 1 FP8 (ROW variant only)
  int act4;       // W4A4: X quantised to NVFP4 in the kernel (MMA variant, staged X)
  int split_k;
  int num_sms;
  size_t ws_bytes;
  nvfp4::GemvConfig gemv;
  nvfp4::TcConfig tc;
  nvfp4::Tc4Config tc4;   // TC variant of a W4A4 plan
  nvfp4::MmaConfig mma;
  nvfp4::RowConfig row;
  std::mutex map_mu;
  MapEntry maps[kMapCache];
  int map_next = 0;
  // mma variant with X in the ring: descriptor of the X planes in the last
  // workspace seen (the planes live in the workspace)
  const void* xmap_ws = nullptr;
  CUtensorMap xmap;
};

namespace {

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

nvfp4_status check_device(int device) {
  int cur = -1;
  if (cudaGetDevice(&cur) != cudaSuccess) return NVFP4_ERR_CUDA;
  return cur == device ? NVFP4_OK : NVFP4_ERR_INVALID_ARG;
}

// Device address of g_static_scratch on `device`, which must be current. The
// first call per device looks it up (this may load the module there).
constexpr int kMaxScratchDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxScratchDevices] = {};

nvfp4_status static_scratch_address(int device, void** out) {
  if (device < 0 || device >= kMaxScratchDevices) return NVFP4_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> g(g_scratch_mu);
  if (!g_scratch_addr[device]) {
    void* a = nullptr;
    if (cudaGetSymbolAddress(&a, g_static_scratch) != cudaSuccess || !a) return NVFP4_ERR_CUDA;
    g_scratch_addr[device] = a;
  }
  *out = g_scratch_addr[device];
  return NVFP4_OK;
}

// Which variant AUTO takes for a shape: the fastest measured variant of the
// nearest shape in the table measured on B200 (variant_table.csv, written
// by tune_variants.py; variant_table.inc is generated from it at build
// time). Nearest: the smallest 2 |log2 M - log2 Mt| + |log2 NK - log2 NtKt|,
// the first such row on a tie. plan() falls back to the MMA pipeline, then
// to tcgen05, when the chosen variant cannot take the shape.
struct TableRow { int M, N, K, variant; };
constexpr TableRow kVariantTable[] = {
#include "variant_table.inc"
};

int auto_variant(int M, int N, int K) {
  if (M < 1 || N < 1 || K < 1) return int(NVFP4_VARIANT_MMA);
  const double lm = std::log2(double(M)), lnk = std::log2(double(N)) + std::log2(double(K));
  double best = 1e300;
  int v = int(NVFP4_VARIANT_MMA);
  for (const TableRow& r : kVariantTable) {
    const double d = 2.0 * std::fabs(lm - std::log2(double(r.M))) +
                     std::fabs(lnk - std::log2(double(r.N)) - std::log2(double(r.K)));
    if (d < best) { best = d; v = r.variant; }
  }
  return v;
}

// Copy of the TMA descriptors for (wp, ws), encoding them on first use.
bool lookup_maps(nvfp4_plan_s* p, const void* wp, const void* ws, CUtensorMap* mw, CUtensorMap* ms) {
  std::lock_guard<std::mutex> g(p->map_mu);
  for (int i = 0; i < kMapCache; ++i) {
    if (p->maps[i].wp == wp && p->maps[i].ws == ws) {
      *mw = p->maps[i].mw;
      *ms = p->maps[i].ms;
      return true;
    }
  }
  MapEntry& e = p->maps[p->map_next];
  bool ok;
  if (p->variant == int(NVFP4_VARIANT_ROW)) {
    ok = nvfp4::encode_row_maps(p->N, p->K, p->row.ipu, p->row.fmt, static_cast<const uint8_t*>(wp),
                                static_cast<const uint8_t*>(ws), &e.mw, &e.ms);
  } else if (p->variant == int(NVFP4_VARIANT_MMA) && p->fmt == 1) {
    // FP8 codes; the row scales are read directly (the second map is unused)
    ok = nvfp4::encode_fp8_codes_map(p->N, p->K, static_cast<const uint8_t*>(wp), &e.mw);
    e.ms = e.mw;
  } else {
    // 256-row boxes for the MMA variant and the W4A4 tensor-core kernel, 128 for TC
    const int box_rows =
        (p->variant == int(NVFP4_VARIANT_MMA) || (p->variant == int(NVFP4_VARIANT_TC) && p->act4))
            ? nvfp4::kMmaTileRows : 128;
    ok = nvfp4::encode_weight_maps(p->N, p->K, box_rows, static_cast<const uint8_t*>(wp),
                                   static_cast<const uint8_t*>(ws), &e.mw, &e.ms);
  }
  if (!ok) {
    e.wp = e.ws = nullptr;
    return false;
  }
  e.wp = wp;
  e.ws = ws;
  p->map_next = (p->map_next + 1) % kMapCache;
  *mw = e.mw;
  *ms = e.ms;
  return true;
}

constexpr long long kTimeoutCycles = 1ll << 31;       // ~1 s at 2 GHz
constexpr long long kStallTimeoutCycles = 1ll << 22;  // test mode: ~2 ms

}  // namespace

extern "C" {

const char* nvfp4_status_string(nvfp4_status s) {
  switch (s) {
    case NVFP4_OK: return "ok";
    case NVFP4_ERR_INVALID_ARG: return "invalid argument";
    case NVFP4_ERR_UNSUPPORTED: return "unsupported shape or variant";
    case NVFP4_ERR_MISALIGNED: return "misaligned pointer";
    case NVFP4_ERR_CUDA: return "CUDA error";
    case NVFP4_ERR_TIMEOUT: return "device wait timed out";
    case NVFP4_ERR_BAD_SCALE: return "bad scale";
    case NVFP4_ERR_WORKSPACE: return "workspace missing or too small";
  }
  return "unknown status";
}

nvfp4_status nvfp4_linear_plan(int M, int N, int K, int device, unsigned flags,
                               nvfp4_plan_t* out) {
  if (!out) return NVFP4_ERR_INVALID_ARG;
  *out = nullptr;
  if (M < 1 || M > 16 || N < 0 || K < 0 || K % 256 != 0) return NVFP4_ERR_INVALID_ARG;
  const unsigned epi_flag = flags & NVFP4_PLAN_EPI_MASK;
  int epi = 0;
  if (epi_flag == NVFP4_PLAN_EPI_SWIGLU) epi = 1;
  else if (epi_flag == NVFP4_PLAN_EPI_ARGMAX) epi = 2;
  else if (epi_flag != 0u) return NVFP4_ERR_INVALID_ARG;
  if (epi == 1 && N % 2 != 0) return NVFP4_ERR_INVALID_ARG;
  const int fmt = (flags & NVFP4_PLAN_WEIGHT_FP8) ? 1 : 0;
  const int act4 = (flags & NVFP4_PLAN_ACT_NVFP4) ? 1 : 0;
  if (act4 && fmt) return NVFP4_ERR_UNSUPPORTED;
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess) return NVFP4_ERR_CUDA;
  if (device < 0 || device >= ndev) return NVFP4_ERR_INVALID_ARG;
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device) != cudaSuccess)
    return NVFP4_ERR_CUDA;
  int prev = -1;
  if (cudaGetDevice(&prev) != cudaSuccess) return NVFP4_ERR_CUDA;
  if (prev != device && cudaSetDevice(device) != cudaSuccess) return NVFP4_ERR_CUDA;

  nvfp4_plan_s* h = new (std::nothrow) nvfp4_plan_s();
  if (!h) { if (prev != device) cudaSetDevice(prev); return NVFP4_ERR_CUDA; }
  nvfp4_plan_s& p = *h;
  p.M = M; p.N = N; p.K = K; p.device = device; p.flags = flags; p.num_sms = sms;
  p.epi = epi;
  p.fmt = fmt;
  p.act4 = act4;
  p.split_k = 1;
  p.ws_bytes = 0;
  unsigned forced = flags & NVFP4_PLAN_VARIANT_MASK;
  // W4A4: the block-scaled FP4 tensor cores from M = 4 on (their time is flat
  // in M), the warp-MMA kernel below that and for the fused epilogues
  p.variant = forced ? int(forced)
              : fmt == 1 ? int(NVFP4_VARIANT_MMA)
              : act4     ? ((M >= 4 && epi == 0) ? int(NVFP4_VARIANT_TC) : int(NVFP4_VARIANT_MMA))
                         : auto_variant(M, N, K);
  if (K == 0 || N == 0) {
    // nothing to contract: run() writes zeros (K == 0) or returns (N == 0)
    if (p.variant == int(NVFP4_VARIANT_GEMV) && M > 4) p.variant = int(NVFP4_VARIANT_TC);
  }
  auto configure = [&]() -> nvfp4_status {
    nvfp4_status st = NVFP4_OK;
    if (p.epi != 0 && p.variant != int(NVFP4_VARIANT_MMA)) return NVFP4_ERR_UNSUPPORTED;
    if (p.fmt != 0 && ((p.variant != int(NVFP4_VARIANT_ROW) && p.variant != int(NVFP4_VARIANT_MMA)) ||
                       p.epi != 0 || p.act4 != 0))
      return NVFP4_ERR_UNSUPPORTED;
    if (p.act4 && p.variant != int(NVFP4_VARIANT_MMA) && p.variant != int(NVFP4_VARIANT_TC))
      return NVFP4_ERR_UNSUPPORTED;
    switch (p.variant) {
      case NVFP4_VARIANT_GEMV: {
        if (M > 4 || size_t(M) * size_t(K) * 4 > 200 * 1024) { st = NVFP4_ERR_UNSUPPORTED; break; }
        p.gemv.M = M; p.gemv.N = N; p.gemv.K = K;
        if (K > 0 && N > 0 && nvfp4::gemv_configure(p.gemv, sms) != cudaSuccess) st = NVFP4_ERR_CUDA;
        break;
      }
      case NVFP4_VARIANT_MMA: {
        if (K == 0 || N == 0) break;
        p.mma.M = M; p.mma.N = N; p.mma.K = K; p.mma.epi = p.epi; p.mma.act4 = p.act4; p.mma.fmt = p.fmt;
        cudaError_t e = nvfp4::mma_configure(p.mma, sms);
        if (e == cudaSuccess && !nvfp4::tensor_maps_supported()) e = cudaErrorNotSupported;
        if (e == cudaErrorInvalidConfiguration || e == cudaErrorNotSupported) st = NVFP4_ERR_UNSUPPORTED;
        else if (e != cudaSuccess) st = NVFP4_ERR_CUDA;
        p.split_k = p.mma.S;
        p.ws_bytes = p.mma.ws_bytes;
        break;
      }
      case NVFP4_VARIANT_ROW: {
        if (K == 0 || N == 0) break;
        p.row.M = M; p.row.N = N; p.row.K = K; p.row.fmt = p.fmt;
        cudaError_t e = nvfp4::row_configure(p.row, sms);
        if (e == cudaSuccess && !nvfp4::tensor_maps_supported()) e = cudaErrorNotSupported;
        if (e == cudaErrorInvalidConfiguration || e == cudaErrorNotSupported) st = NVFP4_ERR_UNSUPPORTED;
        else if (e != cudaSuccess) st = NVFP4_ERR_CUDA;
        p.split_k = p.row.KS;
        p.ws_bytes = p.row.ws_bytes;
        break;
      }
      case NVFP4_VARIANT_TC: {
        if (K == 0 || N == 0) break;
        if (p.act4) {
          p.tc4.M = M; p.tc4.N = N; p.tc4.K = K;
          cudaError_t e = nvfp4::tc4_configure(p.tc4, sms);
          if (e == cudaErrorNotSupported || e == cudaErrorInvalidConfiguration) st = NVFP4_ERR_UNSUPPORTED;
          else if (e != cudaSuccess) st = NVFP4_ERR_CUDA;
          p.split_k = p.tc4.S;
          p.ws_bytes = p.tc4.ws_bytes;
          break;
        }
        p.tc.M = M; p.tc.N = N; p.tc.K = K;
        cudaError_t e = nvfp4::tc_configure(p.tc, sms);
        if (e == cudaErrorNotSupported || e == cudaErrorInvalidConfiguration) st = NVFP4_ERR_UNSUPPORTED;
        else if (e != cudaSuccess) st = NVFP4_ERR_CUDA;
        p.split_k = p.tc.S;
        p.ws_bytes = p.tc.ws_bytes;
        break;
      }
      default:
        st = NVFP4_ERR_UNSUPPORTED;
    }
    return st;
  };
  nvfp4_status st = configure();
  if (st == NVFP4_ERR_UNSUPPORTED && !forced && p.fmt == 1 && p.variant == int(NVFP4_VARIANT_MMA)) {
    // FP8 weights the MMA variant cannot take (X does not fit beside its ring): the row variant
    p.variant = int(NVFP4_VARIANT_ROW);
    p.split_k = 1;
    p.ws_bytes = 0;
    st = configure();
  }
  if (st == NVFP4_ERR_UNSUPPORTED && !forced && p.act4 && p.variant == int(NVFP4_VARIANT_TC)) {
    p.variant = int(NVFP4_VARIANT_MMA);
    p.split_k = 1;
    p.ws_bytes = 0;
    st = configure();
  }
  if (st == NVFP4_ERR_UNSUPPORTED && !forced && p.fmt == 0 && p.variant != int(NVFP4_VARIANT_MMA) &&
      p.variant != int(NVFP4_VARIANT_TC)) {
    // the table's choice (GEMV, row) cannot take this shape or epilogue
    p.variant = int(NVFP4_VARIANT_MMA);
    p.split_k = 1;
    p.ws_bytes = 0;
    st = configure();
  }
  if (st == NVFP4_ERR_UNSUPPORTED && !forced && p.epi == 0 && p.fmt == 0 && p.act4 == 0 &&
      p.variant != int(NVFP4_VARIANT_TC)) {
    // the automatic choice cannot take this shape: the tcgen05 pipeline can
    p.variant = int(NVFP4_VARIANT_TC);
    p.split_k = 1;
    p.ws_bytes = 0;
    st = configure();
  }
  if (prev != device) cudaSetDevice(prev);
  if (st != NVFP4_OK) { delete h; return st; }
  *out = h;
  return NVFP4_OK;
}

int nvfp4_auto_variant(int M, int N, int K) {
  if (M < 1 || M > 16 || N < 0 || K < 0 || K % 256 != 0) return -1;
  return auto_variant(M, N, K);
}

size_t nvfp4_linear_workspace_bytes(nvfp4_plan_t plan) { return plan ? plan->ws_bytes : 0; }
int nvfp4_linear_variant(nvfp4_plan_t plan) { return plan ? plan->variant : -1; }
int nvfp4_linear_split_k(nvfp4_plan_t plan) { return plan ? plan->split_k : -1; }
int nvfp4_linear_launches_per_run(nvfp4_plan_t plan) {
  if (!plan) return -1;
  if (plan->N == 0) return 0;
  if (plan->K > 0 && plan->variant == NVFP4_VARIANT_MMA && plan->mma.xr) return 2;
  if (plan->K > 0 && plan->variant == NVFP4_VARIANT_TC && plan->act4) return 3;
  return 1;
}

void nvfp4_linear_destroy(nvfp4_plan_t plan) { delete plan; }

nvfp4_status nvfp4_linear_run(nvfp4_plan_t plan, const uint8_t* w_packed,
                              const uint8_t* w_scales, const float* w_global,
                              const void* x, void* y, void* workspace, size_t ws_bytes,
                              void* stream) {
  if (!plan) return NVFP4_ERR_INVALID_ARG;
  const int M = plan->M, N = plan->N, K = plan->K;
  if (N == 0) return NVFP4_OK;
  if (!y || !w_global) return NVFP4_ERR_INVALID_ARG;
  if (K > 0 && (!w_packed || !w_scales || !x)) return NVFP4_ERR_INVALID_ARG;
  if (!aligned(y, 16) || !aligned(w_global, 4)) return NVFP4_ERR_MISALIGNED;
  if (K > 0 && (!aligned(w_packed, 16) || !aligned(w_scales, 16) || !aligned(x, 16)))
    return NVFP4_ERR_MISALIGNED;
  if (plan->ws_bytes > 0) {
    if (!workspace || ws_bytes < plan->ws_bytes) return NVFP4_ERR_WORKSPACE;
    if (!aligned(workspace, 16)) return NVFP4_ERR_MISALIGNED;
  }
  nvfp4_status dv = check_device(plan->device);
  if (dv != NVFP4_OK) return dv;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint16_t* yb = static_cast<uint16_t*>(y);
  const uint16_t* xb = static_cast<const uint16_t*>(x);
  cudaError_t e = cudaSuccess;
  if (K == 0) {
    // every sum is zero: Y zero, SwiGLU silu(0) * 0 = 0, argmax row 0 with value 0
    const int64_t count = plan->epi == 1 ? int64_t(M) * (N / 2) : plan->epi == 2 ? 4 * int64_t(M) : int64_t(M) * N;
    e = nvfp4::launch_zero_bf16(yb, count, st);
  } else {
    switch (plan->variant) {
      case NVFP4_VARIANT_GEMV:
        e = nvfp4::launch_gemv(plan->gemv, w_packed, w_scales, w_global, xb, yb, st);
        break;
      case NVFP4_VARIANT_MMA: {
        CUtensorMap mw, ms;
        if (!lookup_maps(plan, w_packed, w_scales, &mw, &ms)) return NVFP4_ERR_CUDA;
        const bool stall = (plan->flags & NVFP4_PLAN_TEST_STALL) != 0;
        const bool pdl = (plan->flags & NVFP4_PLAN_PDL) != 0;
        CUtensorMap mx;
        if (plan->mma.xr) {
          std::lock_guard<std::mutex> g(plan->map_mu);
          if (plan->xmap_ws != workspace) {
            const uint8_t* planes = static_cast<const uint8_t*>(workspace) + plan->mma.ws_x_off;
            if (!nvfp4::encode_x_planes_map(planes, plan->mma.x_pitch, plan->mma.ncols, plan->mma.x_box,
                                            &plan->xmap)) {
              plan->xmap_ws = nullptr;
              return NVFP4_ERR_CUDA;
            }
            plan->xmap_ws = workspace;
          }
          mx = plan->xmap;
        }
        const float* row_scale = plan->fmt == 1 ? static_cast<const float*>(static_cast<const void*>(w_scales)) : nullptr;
        e = nvfp4::launch_mma(plan->mma, &mw, &ms, &mx, w_global, row_scale, xb, yb, workspace,
                              stall ? kStallTimeoutCycles : kTimeoutCycles, stall, pdl, st);
        break;
      }
      case NVFP4_VARIANT_ROW: {
        CUtensorMap mw, ms;
        if (!lookup_maps(plan, w_packed, w_scales, &mw, &ms)) return NVFP4_ERR_CUDA;
        const bool stall = (plan->flags & NVFP4_PLAN_TEST_STALL) != 0;
        const bool pdl = (plan->flags & NVFP4_PLAN_PDL) != 0;
        e = nvfp4::launch_row(plan->row, &mw, &ms, reinterpret_cast<const float*>(w_scales), w_global, xb,
                              yb, workspace,
                              stall ? kStallTimeoutCycles : kTimeoutCycles, stall, pdl, st);
        break;
      }
      case NVFP4_VARIANT_TC: {
        CUtensorMap mw, ms;
        if (!lookup_maps(plan, w_packed, w_scales, &mw, &ms)) return NVFP4_ERR_CUDA;
        const bool stall = (plan->flags & NVFP4_PLAN_TEST_STALL) != 0;
        if (plan->act4) {
          const bool pdl = (plan->flags & NVFP4_PLAN_PDL) != 0;
          e = nvfp4::launch_tc4(plan->tc4, &mw, &ms, w_global, xb, yb, workspace,
                                stall ? kStallTimeoutCycles : kTimeoutCycles, stall, pdl, st);
          break;
        }
        e = nvfp4::launch_tc(plan->tc, &mw, &ms, w_global, xb, yb, workspace,
                             stall ? kStallTimeoutCycles : kTimeoutCycles, stall, st);
        break;
      }
      default:
        return NVFP4_ERR_UNSUPPORTED;
    }
  }
  return e == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}

nvfp4_status nvfp4_linear_status(nvfp4_plan_t plan, void* workspace, void* stream) {
  if (!plan) return NVFP4_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return NVFP4_ERR_CUDA;
  if (cudaPeekAtLastError() != cudaSuccess) return NVFP4_ERR_CUDA;
  if (plan->ws_bytes > 0 && workspace) {
    uint32_t word = 0;
    if (cudaMemcpy(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess)
      return NVFP4_ERR_CUDA;
    if (word != 0) {
      // an aborted run can leave split counters behind: clear the whole workspace
      if (cudaMemset(workspace, 0, plan->ws_bytes) != cudaSuccess) return NVFP4_ERR_CUDA;
      if (cudaDeviceSynchronize() != cudaSuccess) return NVFP4_ERR_CUDA;
      return NVFP4_ERR_TIMEOUT;
    }
  }
  return NVFP4_OK;
}

nvfp4_status nvfp4_pack_check(const uint8_t* w_packed, const uint8_t* w_scales,
                              const float* w_global, int N, int K, void* w_bf16_out,
                              unsigned* d_bad, void* stream) {
  if (N < 0 || K < 0 || K % 16 != 0) return NVFP4_ERR_INVALID_ARG;
  if (!w_global || !d_bad) return NVFP4_ERR_INVALID_ARG;
  const int64_t nb = int64_t(N) * (K / 16);
  if (nb > 0 && (!w_packed || !w_scales)) return NVFP4_ERR_INVALID_ARG;
  if (!aligned(w_global, 4) || !aligned(d_bad, 4)) return NVFP4_ERR_MISALIGNED;
  if (nb > 0 && (!aligned(w_packed, 16) || !aligned(w_scales, 16))) return NVFP4_ERR_MISALIGNED;
  if (w_bf16_out && !aligned(w_bf16_out, 16)) return NVFP4_ERR_MISALIGNED;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return NVFP4_ERR_CUDA;
  cudaError_t e = nvfp4::launch_pack_check(w_packed, w_scales, w_global, nb,
                                           static_cast<uint16_t*>(w_bf16_out), d_bad, sms,
                                           static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}

nvfp4_status nvfp4_quantize(const float* w, int N, int K, uint8_t* w_packed, uint8_t* w_scales,
                            float* w_global, unsigned* d_bad, void* stream) {
  if (N < 0 || K < 0 || K % 16 != 0 || !w_global) return NVFP4_ERR_INVALID_ARG;
  const int64_t n = int64_t(N) * K;
  if (n > 0 && (!w || !w_packed || !w_scales)) return NVFP4_ERR_INVALID_ARG;
  if (!aligned(w_global, 4) || (d_bad && !aligned(d_bad, 4))) return NVFP4_ERR_MISALIGNED;
  if (n > 0 && (!aligned(w, 16) || !aligned(w_packed, 16) || !aligned(w_scales, 16)))
    return NVFP4_ERR_MISALIGNED;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return NVFP4_ERR_CUDA;
  cudaError_t e = nvfp4::launch_quantize(w, N, K, w_packed, w_scales, w_global, d_bad, sms,
                                         static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}

nvfp4_status nvfp4_quantize_fp8(const float* w, int N, int K, uint8_t* codes, float* row_scales,
                                unsigned* d_bad, void* stream) {
  if (N < 0 || K < 0 || K % 16 != 0) return NVFP4_ERR_INVALID_ARG;
  if (N > 0 && !row_scales) return NVFP4_ERR_INVALID_ARG;
  const int64_t n = int64_t(N) * K;
  if (n > 0 && (!w || !codes)) return NVFP4_ERR_INVALID_ARG;
  if ((d_bad && !aligned(d_bad, 4)) || (N > 0 && !aligned(row_scales, 16))) return NVFP4_ERR_MISALIGNED;
  if (n > 0 && (!aligned(w, 16) || !aligned(codes, 16))) return NVFP4_ERR_MISALIGNED;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return NVFP4_ERR_CUDA;
  cudaError_t e = nvfp4::launch_quantize_fp8(w, N, K, codes, row_scales, d_bad, sms,
                                             static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}

nvfp4_status nvfp4_linear_run_static(nvfp4_plan_t plan, const uint8_t* w_packed,
                                     const uint8_t* w_scales, const float* w_global,
                                     const void* x, void* y, unsigned* status_out,
                                     void* stream) {
  if (!plan) return NVFP4_ERR_INVALID_ARG;
  if (plan->ws_bytes > size_t(NVFP4_STATIC_SCRATCH_BYTES)) return NVFP4_ERR_WORKSPACE;
  if (status_out && !aligned(status_out, 4)) return NVFP4_ERR_MISALIGNED;
  nvfp4_status s = check_device(plan->device);
  if (s != NVFP4_OK) return s;
  void* scratch = nullptr;
  s = static_scratch_address(plan->device, &scratch);
  if (s != NVFP4_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // Status word and per-tile counters must start at zero; the partial sums
  // are written before they are read.
  size_t zeroed = plan->ws_bytes;
  if (plan->variant == int(NVFP4_VARIANT_MMA) && plan->mma.ws_partials_off < zeroed)
    zeroed = plan->mma.ws_partials_off;
  if (plan->variant == int(NVFP4_VARIANT_TC) && !plan->act4 && plan->tc.ws_partials_off < zeroed)
    zeroed = plan->tc.ws_partials_off;
  // W4A4 on the FP4 tensor cores: status word, X amax, gs_x and counters lie
  // before the X blocks
  if (plan->variant == int(NVFP4_VARIANT_TC) && plan->act4 && plan->tc4.ws_x_off < zeroed)
    zeroed = plan->tc4.ws_x_off;
  if (plan->variant == int(NVFP4_VARIANT_ROW) && plan->row.ws_partials_off < zeroed)
    zeroed = plan->row.ws_partials_off;
  if (zeroed > 0 && cudaMemsetAsync(scratch, 0, zeroed, st) != cudaSuccess) return NVFP4_ERR_CUDA;
  s = nvfp4_linear_run(plan, w_packed, w_scales, w_global, x, y, scratch,
                       size_t(NVFP4_STATIC_SCRATCH_BYTES), stream);
  if (s != NVFP4_OK) return s;
  if (status_out) {
    const cudaError_t e = plan->ws_bytes > 0
        ? cudaMemcpyAsync(status_out, scratch, sizeof(unsigned), cudaMemcpyDeviceToDevice, st)
        : cudaMemsetAsync(status_out, 0, sizeof(unsigned), st);
    if (e != cudaSuccess) return NVFP4_ERR_CUDA;
  }
  return NVFP4_OK;
}

}  // extern "C"
