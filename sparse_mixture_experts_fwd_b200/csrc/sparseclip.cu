// SparseClip global gradient norm ("[Paper review] TorchScale: Transformers
// at Scale", proposed method):
//   ||g||_2 = ||(g_d, kappa g_s)||_2 = sqrt(Sd + kappa^2 Ss),  kappa = 1/sqrt(E)
// where Sd / Ss are the sums of squares of the dense / expert gradients, and
// the clipping step that uses it: every gradient scaled by
// min(1, max_norm / ||g||_2).
//
// One bandwidth pass: a fixed grid of kGrid blocks streams every tensor with
// 16-byte loads (4 in flight per thread), squares and sums each float4 in
// fp32, accumulates those in fp64 per thread, reduces per block in a fixed
// shuffle/shared-memory order and writes one fp64 partial per (launch, block,
// class).  A one-block kernel then sums the partials in a fixed order, so the
// result does not depend on scheduling.  Segments go to the kernel by value
// (kSegsPerLaunch per launch), so no host->device copy is needed.
#include <algorithm>
#include <cmath>
#include <mutex>
#include <vector>

#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int kGrid = 1024;
constexpr int kBlock = 256;
constexpr int kSegsPerLaunch = 128;
constexpr int kMaxSegs = 4096;

struct ClipSeg {
  const float* ptr;
  int64_t len;
  int32_t cls;  // 0 dense, 1 expert
  int32_t pad;
};
struct ClipBatch {
  ClipSeg seg[kSegsPerLaunch];
  int32_t n;
};

__device__ __forceinline__ double block_sum(double v, double* s_red) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_down_sync(0xffffffffu, v, off);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane == 0) s_red[warp] = v;
  __syncthreads();
  double r = 0.0;
  if (threadIdx.x == 0)
    for (int w = 0; w < kBlock / 32; ++w) r += s_red[w];
  __syncthreads();
  return r;  // valid in thread 0
}

__device__ __forceinline__ float sq4(const float4& v) {
  return v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
}

__global__ void __launch_bounds__(kBlock) sumsq_kernel(const ClipBatch b, double* partials) {
  __shared__ double s_red[kBlock / 32];
  double acc_d = 0.0, acc_e = 0.0;  // dense, expert
  const int64_t gtid = static_cast<int64_t>(blockIdx.x) * kBlock + threadIdx.x;
  const int64_t nth = static_cast<int64_t>(gridDim.x) * kBlock;
  for (int s = 0; s < b.n; ++s) {
    const float* p = b.seg[s].ptr;
    const int64_t n = b.seg[s].len;
    const int64_t n4 = n >> 2;
    const float4* p4 = reinterpret_cast<const float4*>(p);
    double a = 0.0;
    int64_t i = gtid;
    for (; i + 3 * nth < n4; i += 4 * nth) {
      const float4 v0 = __ldg(p4 + i);
      const float4 v1 = __ldg(p4 + i + nth);
      const float4 v2 = __ldg(p4 + i + 2 * nth);
      const float4 v3 = __ldg(p4 + i + 3 * nth);
      a += static_cast<double>(sq4(v0));
      a += static_cast<double>(sq4(v1));
      a += static_cast<double>(sq4(v2));
      a += static_cast<double>(sq4(v3));
    }
    for (; i < n4; i += nth) a += static_cast<double>(sq4(__ldg(p4 + i)));
    for (int64_t j = 4 * n4 + gtid; j < n; j += nth) {
      const float v = __ldg(p + j);
      a += static_cast<double>(v * v);
    }
    if (b.seg[s].cls) acc_e += a; else acc_d += a;
  }
  const double d = block_sum(acc_d, s_red);
  const double e = block_sum(acc_e, s_red);
  if (threadIdx.x == 0) {
    partials[2 * blockIdx.x] = d;
    partials[2 * blockIdx.x + 1] = e;
  }
}

__global__ void __launch_bounds__(kBlock) finish_kernel(const double* partials, int n_partials,
                                                        int num_experts, double* out) {
  __shared__ double s_red[kBlock / 32];
  double a = 0.0, e = 0.0;
  for (int i = threadIdx.x; i < n_partials; i += kBlock) {
    a += partials[2 * i];
    e += partials[2 * i + 1];
  }
  const double sd = block_sum(a, s_red);
  const double ss = block_sum(e, s_red);
  if (threadIdx.x == 0) {
    out[0] = sqrt(sd + ss / static_cast<double>(num_experts));  // kappa^2 = 1/E
    out[1] = sd;
    out[2] = ss;
  }
}

// Clipping step: every tensor (dense and expert) scaled in place by
// coef = min(1, max_norm / norm), norm = out[0] written by finish_kernel on
// the same stream.  When coef is 1 nothing is written.  Block 0 records coef
// in out[3].  16-byte loads and stores, the same grid-stride order as the sum.
struct ScaleSeg {
  float* ptr;
  int64_t len;
};
struct ScaleBatch {
  ScaleSeg seg[kSegsPerLaunch];
  int32_t n;
};

__global__ void __launch_bounds__(kBlock) scale_kernel(const ScaleBatch b, double max_norm,
                                                       double* out, int write_coef) {
  const double norm = out[0];
  const double coefd = norm > max_norm ? max_norm / norm : 1.0;
  if (write_coef && blockIdx.x == 0 && threadIdx.x == 0) out[3] = coefd;
  if (coefd == 1.0) return;
  const float c = static_cast<float>(coefd);
  const int64_t gtid = static_cast<int64_t>(blockIdx.x) * kBlock + threadIdx.x;
  const int64_t nth = static_cast<int64_t>(gridDim.x) * kBlock;
  for (int s = 0; s < b.n; ++s) {
    float* p = b.seg[s].ptr;
    const int64_t n = b.seg[s].len;
    const int64_t n4 = n >> 2;
    float4* p4 = reinterpret_cast<float4*>(p);
    int64_t i = gtid;
    for (; i + nth < n4; i += 2 * nth) {
      float4 v0 = p4[i];
      float4 v1 = p4[i + nth];
      v0.x *= c; v0.y *= c; v0.z *= c; v0.w *= c;
      v1.x *= c; v1.y *= c; v1.z *= c; v1.w *= c;
      p4[i] = v0;
      p4[i + nth] = v1;
    }
    for (; i < n4; i += nth) {
      float4 v = p4[i];
      v.x *= c; v.y *= c; v.z *= c; v.w *= c;
      p4[i] = v;
    }
    for (int64_t j = 4 * n4 + gtid; j < n; j += nth) p[j] *= c;
  }
}

int64_t n_launches(int32_t n_dense, int32_t n_sparse) {
  const int64_t n = static_cast<int64_t>(n_dense) + n_sparse;
  return std::max<int64_t>(1, (n + kSegsPerLaunch - 1) / kSegsPerLaunch);
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" size_t sparseclip_workspace_size(int32_t n_dense, int32_t n_sparse) {
  if (n_dense < 0 || n_sparse < 0 || static_cast<int64_t>(n_dense) + n_sparse > kMaxSegs) return 0;
  return static_cast<size_t>(n_launches(n_dense, n_sparse)) * kGrid * 2 * sizeof(double);
}

extern "C" int32_t sparseclip_norm(const float* const* dense, const int64_t* dense_len,
                                   int32_t n_dense, const float* const* sparse,
                                   const int64_t* sparse_len, int32_t n_sparse,
                                   int32_t num_experts, double* out, void* workspace,
                                   size_t workspace_bytes, moe_stream_t stream) {
  CallRange range_("sparseclip_norm");
  set_last_error("");
  if (n_dense < 0 || n_sparse < 0 || static_cast<int64_t>(n_dense) + n_sparse > kMaxSegs)
    return fail(MOE_ERR_INVALID_ARGUMENT, "sparseclip_norm: segment counts out of range");
  if ((n_dense > 0 && (!dense || !dense_len)) || (n_sparse > 0 && (!sparse || !sparse_len)))
    return fail(MOE_ERR_INVALID_ARGUMENT, "sparseclip_norm: null segment array");
  if (num_experts < 1) return fail(MOE_ERR_INVALID_ARGUMENT, "sparseclip_norm: num_experts < 1");
  if (!out) return fail(MOE_ERR_INVALID_ARGUMENT, "sparseclip_norm: null out");
  const size_t need = sparseclip_workspace_size(n_dense, n_sparse);
  if (!workspace || workspace_bytes < need)
    return fail(MOE_ERR_WORKSPACE, "sparseclip_norm: workspace needs " + std::to_string(need) +
                                       " bytes");
  if (!aligned16(workspace)) return fail(MOE_ERR_ALIGNMENT, "sparseclip_norm: workspace");
  std::vector<ClipSeg> segs;
  for (int pass = 0; pass < 2; ++pass) {
    const int32_t n = pass == 0 ? n_dense : n_sparse;
    const float* const* ptrs = pass == 0 ? dense : sparse;
    const int64_t* lens = pass == 0 ? dense_len : sparse_len;
    for (int32_t i = 0; i < n; ++i) {
      if (lens[i] < 0) return fail(MOE_ERR_INVALID_ARGUMENT, "sparseclip_norm: negative length");
      if (lens[i] == 0) continue;
      if (!ptrs[i]) return fail(MOE_ERR_INVALID_ARGUMENT, "sparseclip_norm: null tensor");
      if (!aligned16(ptrs[i])) return fail(MOE_ERR_ALIGNMENT, "sparseclip_norm: tensor not 16-byte aligned");
      segs.push_back(ClipSeg{ptrs[i], lens[i], pass, 0});
    }
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  double* partials = static_cast<double*>(workspace);
  const int64_t launches = std::max<int64_t>(1, (static_cast<int64_t>(segs.size()) + kSegsPerLaunch - 1) / kSegsPerLaunch);
  for (int64_t l = 0; l < launches; ++l) {
    ClipBatch b{};
    const size_t first = static_cast<size_t>(l) * kSegsPerLaunch;
    b.n = static_cast<int32_t>(std::min<size_t>(kSegsPerLaunch, segs.size() - std::min(first, segs.size())));
    for (int32_t i = 0; i < b.n; ++i) b.seg[i] = segs[first + i];
    sumsq_kernel<<<kGrid, kBlock, 0, s>>>(b, partials + l * kGrid * 2);
    int32_t rc = check_launch("sumsq_kernel");
    if (rc != MOE_OK) return rc;
  }
  finish_kernel<<<1, kBlock, 0, s>>>(partials, static_cast<int>(launches * kGrid), num_experts, out);
  return check_launch("finish_kernel");
}

extern "C" int32_t sparseclip_clip(float* const* dense, const int64_t* dense_len, int32_t n_dense,
                                   float* const* sparse, const int64_t* sparse_len,
                                   int32_t n_sparse, int32_t num_experts, double max_norm,
                                   double* out, void* workspace, size_t workspace_bytes,
                                   moe_stream_t stream) {
  CallRange range_("sparseclip_clip");
  set_last_error("");
  if (!(max_norm > 0.0) || !std::isfinite(max_norm))
    return fail(MOE_ERR_INVALID_ARGUMENT, "sparseclip_clip: max_norm must be positive and finite");
  // the norm first (validates every argument), into out[0..2]
  int32_t rc = sparseclip_norm(dense, dense_len, n_dense, sparse, sparse_len, n_sparse,
                               num_experts, out, workspace, workspace_bytes, stream);
  if (rc != MOE_OK) return rc;
  std::vector<ScaleSeg> segs;
  for (int pass = 0; pass < 2; ++pass) {
    const int32_t n = pass == 0 ? n_dense : n_sparse;
    float* const* ptrs = pass == 0 ? dense : sparse;
    const int64_t* lens = pass == 0 ? dense_len : sparse_len;
    for (int32_t i = 0; i < n; ++i)
      if (lens[i] > 0) segs.push_back(ScaleSeg{ptrs[i], lens[i]});
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int64_t launches =
      std::max<int64_t>(1, (static_cast<int64_t>(segs.size()) + kSegsPerLaunch - 1) / kSegsPerLaunch);
  for (int64_t l = 0; l < launches; ++l) {
    ScaleBatch b{};
    const size_t first = static_cast<size_t>(l) * kSegsPerLaunch;
    b.n = static_cast<int32_t>(std::min<size_t>(kSegsPerLaunch, segs.size() - std::min(first, segs.size())));
    for (int32_t i = 0; i < b.n; ++i) b.seg[i] = segs[first + i];
    scale_kernel<<<kGrid, kBlock, 0, s>>>(b, max_norm, out, l == 0 ? 1 : 0);
    rc = check_launch("scale_kernel");
    if (rc != MOE_OK) return rc;
  }
  return MOE_OK;
}

// ---------------------------------------------------------------------------
// No-allocation variant.
//
// Some callers cannot hand the library a workspace: a process whose device
// memory is carved up once at start-up by its own pool (a serving or
// training runtime that forbids allocation on its hot path), or code running
// where calling the CUDA allocator is not allowed or would interfere with
// the caller's allocator (allocator callbacks, out-of-memory recovery).
// sparseclip_norm_noalloc keeps its per-block partial sums in a fixed array
// in the library's own device memory instead.  The array is 128 KiB and
// exists on every GPU that loads the library until the process exits; it
// bounds the call to kStaticMaxSegs tensors.  Every call writes each partial
// it later reads, so nothing needs clearing between calls, but all calls on a
// device share the array: calls that overlap on the GPU (other streams,
// other host threads) race and must be serialised by the caller.
// ---------------------------------------------------------------------------

namespace moe {
namespace {

constexpr int kStaticMaxSegs = 1024;
constexpr int kStaticMaxLaunches = kStaticMaxSegs / kSegsPerLaunch;

static __device__ __align__(256) double g_static_partials[kStaticMaxLaunches * kGrid * 2];

std::mutex g_static_mu;
// The array's address belongs to one CUDA context: it is looked up with the
// device current and cached per (device, context), so a caller that switches
// to another context on the device (or resets the device) gets a fresh lookup.
struct StaticAddr {
  CUcontext ctx;
  double* ptr;
};
StaticAddr g_static_addr[64] = {};

using CtxGetCurrentFn = CUresult (*)(CUcontext*);

CtxGetCurrentFn ctx_get_current_fn() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(ptr);
  });
  return fn;
}

// Device address of g_static_partials in the current context, looked up with
// cudaGetSymbolAddress on the first call made with each device / context
// current (so that first call should come before any stream capture).
int32_t static_partials(double** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(MOE_ERR_CUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
  if (dev < 0 || dev >= 64) return fail(MOE_ERR_UNSUPPORTED, "device ordinal >= 64");
  CtxGetCurrentFn get = ctx_get_current_fn();
  if (!get) return fail(MOE_ERR_CUDA, "cuCtxGetCurrent unavailable from the driver");
  CUcontext ctx = nullptr;  // null before the runtime has made a context current
  if (get(&ctx) != CUDA_SUCCESS) return fail(MOE_ERR_CUDA, "cuCtxGetCurrent failed");
  std::lock_guard<std::mutex> lock(g_static_mu);
  StaticAddr& a = g_static_addr[dev];
  if (!ctx || !a.ptr || a.ctx != ctx) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_partials);  // makes the device's context current
    if (e != cudaSuccess || !p)
      return fail(MOE_ERR_CUDA, std::string("cudaGetSymbolAddress: ") + cudaGetErrorString(e));
    if (get(&ctx) != CUDA_SUCCESS || !ctx) return fail(MOE_ERR_CUDA, "cuCtxGetCurrent failed");
    a.ctx = ctx;
    a.ptr = static_cast<double*>(p);
  }
  *out = a.ptr;
  return MOE_OK;
}

}  // namespace
}  // namespace moe

extern "C" int32_t sparseclip_norm_noalloc(const float* const* dense, const int64_t* dense_len,
                                           int32_t n_dense, const float* const* sparse,
                                           const int64_t* sparse_len, int32_t n_sparse,
                                           int32_t num_experts, double* out, moe_stream_t stream) {
  set_last_error("");
  if (n_dense < 0 || n_sparse < 0)
    return fail(MOE_ERR_INVALID_ARGUMENT, "sparseclip_norm_noalloc: negative segment count");
  if (static_cast<int64_t>(n_dense) + n_sparse > kStaticMaxSegs)
    return fail(MOE_ERR_UNSUPPORTED, "sparseclip_norm_noalloc: at most " +
                                         std::to_string(kStaticMaxSegs) +
                                         " tensors (n_dense + n_sparse) per call");
  if ((n_dense > 0 && (!dense || !dense_len)) || (n_sparse > 0 && (!sparse || !sparse_len)))
    return fail(MOE_ERR_INVALID_ARGUMENT, "sparseclip_norm_noalloc: null segment array");
  if (num_experts < 1)
    return fail(MOE_ERR_INVALID_ARGUMENT, "sparseclip_norm_noalloc: num_experts < 1");
  if (!out) return fail(MOE_ERR_INVALID_ARGUMENT, "sparseclip_norm_noalloc: null out");
  std::vector<ClipSeg> segs;
  for (int pass = 0; pass < 2; ++pass) {
    const int32_t n = pass == 0 ? n_dense : n_sparse;
    const float* const* ptrs = pass == 0 ? dense : sparse;
    const int64_t* lens = pass == 0 ? dense_len : sparse_len;
    for (int32_t i = 0; i < n; ++i) {
      if (lens[i] < 0)
        return fail(MOE_ERR_INVALID_ARGUMENT, "sparseclip_norm_noalloc: negative length");
      if (lens[i] == 0) continue;
      if (!ptrs[i]) return fail(MOE_ERR_INVALID_ARGUMENT, "sparseclip_norm_noalloc: null tensor");
      if (!aligned16(ptrs[i]))
        return fail(MOE_ERR_ALIGNMENT, "sparseclip_norm_noalloc: tensor not 16-byte aligned");
      segs.push_back(ClipSeg{ptrs[i], lens[i], pass, 0});
    }
  }
  double* partials = nullptr;
  int32_t rc = static_partials(&partials);
  if (rc != MOE_OK) return rc;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int64_t launches =
      std::max<int64_t>(1, (static_cast<int64_t>(segs.size()) + kSegsPerLaunch - 1) / kSegsPerLaunch);
  for (int64_t l = 0; l < launches; ++l) {
    ClipBatch b{};
    const size_t first = static_cast<size_t>(l) * kSegsPerLaunch;
    b.n = static_cast<int32_t>(std::min<size_t>(kSegsPerLaunch, segs.size() - std::min(first, segs.size())));
    for (int32_t i = 0; i < b.n; ++i) b.seg[i] = segs[first + i];
    sumsq_kernel<<<kGrid, kBlock, 0, s>>>(b, partials + l * kGrid * 2);
    rc = check_launch("sumsq_kernel (no-alloc)");
    if (rc != MOE_OK) return rc;
  }
  finish_kernel<<<1, kBlock, 0, s>>>(partials, static_cast<int>(launches * kGrid), num_experts, out);
  return check_launch("finish_kernel (no-alloc)");
}
