// Internal helpers shared by the library's translation units: error
// plumbing, launch geometry and the sm_100a PTX wrappers (mbarrier, TMA,
// tcgen05) used by the tensor-core kernels.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <cstdint>
#include <string>

#include "../../include/moe_b200.h"

// 1: dispatch and combine check every expert index and slot they read
// (the libmoe_b200_checked.so build); 0: they trust them.
#ifndef MOE_CHECK_BOUNDS
#define MOE_CHECK_BOUNDS 0
#endif

namespace moe {

// ---- host-side error helpers ------------------------------------------------

void set_last_error(const std::string& msg);
const char* last_error_cstr();
int32_t fail(int32_t code, const std::string& msg);
int32_t check_launch(const char* what);  // maps cudaGetLastError to MOE_ERR_CUDA
int num_sms();                            // SM count of the current device (cached)
uint64_t wait_limit_ns();                 // limit of every bounded wait, for the next launches

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// A named NVTX range around one C-ABI call (host side: from entry to return,
// i.e. validation and enqueueing), so a profiler's timeline shows which call
// launched which kernels and `ncu --nvtx --nvtx-include` can select them.
// Without an attached tool it costs one branch.
struct CallRange {
  explicit CallRange(const char* name) { nvtxRangePushA(name); }
  ~CallRange() { nvtxRangePop(); }
  CallRange(const CallRange&) = delete;
  CallRange& operator=(const CallRange&) = delete;
};

// Launch `kern` with programmatic stream serialisation (see pdl_wait).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t s, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}
inline size_t elem_size(int32_t dtype) { return dtype == MOE_DTYPE_BF16 ? 2 : 4; }
inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

// ---- internal launchers (defined in the .cu files) ---------------------------

// 2-D bf16 [rows, cols] tensor map, boxes of box_rows x 64 (128-byte swizzle)
int32_t make_tmap_bf16(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                       uint32_t box_rows);
int32_t launch_router_tc(const moe_config& c, const void* x, const void* Wr, const float* bias,
                         float* logits, int32_t* status, cudaStream_t s);
int32_t launch_router_f32(const moe_config& c, const void* x, const void* Wr, const float* bias,
                          float* logits, cudaStream_t s);
// Top-1 layers: the expert FFN's second GEMM writes y[t] = gate[t] * E(x_t)
// directly in token order (row -> token map tok_of_row) instead of ye.
struct Top1Out {
  const int32_t* tok_of_row;
  const float* gate;
  void* y;
};
int32_t launch_ffn_two_pass(const moe_config& c, const void* xe, const void* W1, const void* W2,
                            const int32_t* kept_cnt, void* H, void* ye, int32_t* status,
                            cudaStream_t s, const Top1Out* top1 = nullptr);
int32_t launch_ffn_pairs(const moe_config& c, const void* xe, const void* W1, const void* W2,
                         const int32_t* kept_cnt, void* H, void* ye, int32_t* status,
                         cudaStream_t s, const Top1Out* top1 = nullptr);
// sync: ffn_sync_bytes(c) bytes of scratch; sync_zeroed says the caller
// already zeroed it on this stream (else the launcher does).
size_t ffn_sync_bytes(const moe_config& c);
int32_t launch_ffn_tc(const moe_config& c, const void* xe, const void* W1, const void* W2,
                      const int32_t* kept_cnt, void* H, void* ye, void* sync, bool sync_zeroed,
                      int32_t* status, cudaStream_t s, const Top1Out* top1 = nullptr);
// C >= 512: both GEMMs in one persistent launch on SM pairs; sync as above
// (ffn_sync_bytes), chunks of at most 256 rows per expert
int ffn_pair_chunks(const moe_config& c);
int32_t launch_ffn_pair_fused(const moe_config& c, const void* xe, const void* W1, const void* W2,
                              const int32_t* kept_cnt, void* H, void* ye, void* sync,
                              bool sync_zeroed, int32_t* status, cudaStream_t s,
                              const Top1Out* top1 = nullptr);
int32_t launch_ffn_f32(const moe_config& c, const void* xe, const void* W1, const void* W2,
                       const int32_t* kept_cnt, void* H, void* ye, cudaStream_t s);
int32_t launch_route_assign(const moe_config& c, const float* logits, const int32_t* domain,
                            int32_t* expert_idx, float* gate, int32_t* slot, uint8_t* kept,
                            int32_t* tok_of_row, int32_t* arrivals, int32_t* kept_cnt,
                            int32_t* n_dropped, void* scratch, int32_t* status,
                            cudaStream_t s);
size_t assign_scratch_bytes(const moe_config& c);
int32_t launch_router_topk_tc(const moe_config& c, const void* x, const void* Wr,
                              const float* bias, int32_t* expert_idx, float* gate,
                              int32_t* status, cudaStream_t s);
int32_t launch_assign(const moe_config& c, const int32_t* expert_idx, int32_t* slot,
                      uint8_t* kept, int32_t* tok_of_row, int32_t* arrivals, int32_t* kept_cnt,
                      int32_t* n_dropped, void* scratch, int32_t* status, cudaStream_t s);
// zero_words (nullable): n_zero words the dispatch kernel clears for the next kernel;
// y_zero (nullable): y [T, d], whose rows of tokens with no kept choice it zeroes
int32_t launch_dispatch(const moe_config& c, const void* x, const int32_t* expert_idx,
                        const int32_t* slot, const uint8_t* kept, void* xe, int32_t* status,
                        cudaStream_t s,
                        unsigned int* zero_words = nullptr, int n_zero = 0,
                        void* y_zero = nullptr);
// Switch load-balancing loss (eqs. 4-6) and routing entropy from logits [T, E]
size_t aux_workspace_bytes(const moe_config& c);
int32_t launch_aux_loss(const moe_config& c, const float* logits, double alpha, double* out,
                        double* f, double* P, void* workspace, cudaStream_t s);
int32_t launch_combine(const moe_config& c, const void* ye, const int32_t* expert_idx,
                       const float* gate, const int32_t* slot, const uint8_t* kept, void* y,
                       int32_t* status, cudaStream_t s);
// expert parallelism over the ranks of one node: the receive buffers of all
// ranks as mapped into this process, rank order
constexpr int kMaxEpRanks = 8;
int32_t launch_ep_dispatch(const moe_config& c, int rank, int world, const void* x,
                           const int32_t* expert_idx, const int32_t* slot, const uint8_t* kept,
                           const int32_t* cnt_all, void* const* xe_peers, int32_t* local_cnt,
                           int32_t* status, cudaStream_t s);
int32_t launch_ep_combine(const moe_config& c, int rank, int world, const void* const* ye_peers,
                          const int32_t* expert_idx, const float* gate, const int32_t* slot,
                          const uint8_t* kept, const int32_t* cnt_all, void* y, int32_t* status,
                          cudaStream_t s);

}  // namespace moe

// ---- device-side helpers -----------------------------------------------------

#define MOE_DEV __device__ __forceinline__

namespace moe {
namespace dev {

// Wall-clock limit of every spin-wait in the library's kernels, unless the
// host sets another with moe_set_wait_limit_ns (kernels take it as a parameter).
constexpr unsigned long long kDefaultWaitLimitNs = 1000000000ull;  // 1 s

MOE_DEV unsigned long long globaltimer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// The give-up signal that all bounded waits of a kernel share.  `status` is
// the call's status word: its MOE_STATUS_TIMEOUT bit, once any CTA of any
// kernel of the call sets it, makes every other wait of the call give up at
// its next poll, so one expired wait ends the whole grid (and the kernels
// after it on the stream) within about one poll interval instead of each
// CTA spending its own limit.  `local` is the CTA's own flag, the only
// signal when the caller passed no status word.
struct Abort {
  volatile int* local;
  int32_t* status;
  unsigned long long limit_ns;

  MOE_DEV bool raised() const {
    if (*local) return true;
    return status && (*reinterpret_cast<volatile int32_t*>(status) & MOE_STATUS_TIMEOUT);
  }
  // The CTA's own flag only: a shared-memory read, for the per-tile checks of
  // producer and MMA loops (the status word is a global-memory round trip;
  // the bounded waits poll it)
  MOE_DEV bool raised_here() const { return *local != 0; }
  MOE_DEV void raise() const {
    *local = 1;
    if (status) atomicOr(status, MOE_STATUS_TIMEOUT);
  }
};

MOE_DEV uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

MOE_DEV uint32_t lane_id() { return threadIdx.x & 31u; }

// Programmatic dependent launch.  Every kernel of the library is launched
// with programmatic stream serialisation: it lets the next kernel start
// early (pdl_trigger at entry) and performs pdl_wait, which returns once the
// previous kernel on the stream has completed and its writes are visible,
// before its first global-memory read or write.  Tensor memory is allocated
// only after pdl_wait: a CTA that took TMEM before it and landed on an SM
// whose CTA of the previous kernel had triggered but not yet allocated
// would block that allocation (tcgen05.alloc waits for free columns) while
// itself waiting for that kernel to finish.
MOE_DEV void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
MOE_DEV void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// -- mbarrier --
MOE_DEV void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}
MOE_DEV void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
MOE_DEV void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
MOE_DEV void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
MOE_DEV bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Wait for the phase of `parity` to complete, for at most ab.limit_ns, or
// until the give-up signal is raised.  False on timeout / give-up; a timeout
// raises the signal (sets the CTA flag and the status word's timeout bit).
MOE_DEV bool mbar_wait(uint64_t* bar, uint32_t parity, const Abort& ab) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0) {
      if (ab.raised()) return false;
      if (globaltimer() - t0 > ab.limit_ns) {
        ab.raise();
        return false;
      }
    }
  }
}
// The waits a CTA makes before it exits, for copies and MMAs it has already
// issued: they ignore the give-up signal (the hardware is still writing this
// CTA's shared memory or tensor memory) and share one absolute deadline, so
// the whole drain takes at most one limit.
MOE_DEV bool mbar_wait_drain(uint64_t* bar, uint32_t parity, const Abort& ab,
                             unsigned long long deadline) {
  for (uint32_t it = 0;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 63u && globaltimer() > deadline) {
      ab.raise();
      return false;
    }
  }
}

// -- TMA (every load fills the issuing CTA's own shared memory) --
MOE_DEV void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}
MOE_DEV void tma_load_2d(void* smem_dst, const CUtensorMap* map, uint64_t* bar, int32_t x,
                         int32_t y, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "l"(policy)
      : "memory");
}
MOE_DEV void tma_load_2d(void* smem_dst, const CUtensorMap* map, uint64_t* bar, int32_t x,
                         int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}
MOE_DEV uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
MOE_DEV uint64_t policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// -- tcgen05 (cta_group::1) --
MOE_DEV void tmem_alloc(uint32_t* smem_dst, uint32_t ncols) {  // whole warp
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(smem_dst)),
               "r"(ncols)
               : "memory");
}
MOE_DEV void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
MOE_DEV void tmem_dealloc(uint32_t taddr, uint32_t ncols) {  // whole warp
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
MOE_DEV void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
MOE_DEV void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A[smem] * B[smem]^T, kind::f16 (bf16 inputs, fp32 accumulate)
MOE_DEV void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive once on `bar` when every tcgen05.mma issued so far by this thread completes.
MOE_DEV void umma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}
// -- SM pairs (thread-block clusters of two CTAs, tcgen05 cta_group::2) --
MOE_DEV uint32_t cta_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
MOE_DEV void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}
// shared::cluster address of `p` (a shared variable) in CTA `rank` of the cluster
MOE_DEV uint32_t mapa(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}
MOE_DEV void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}
MOE_DEV void st_cluster_u32(uint32_t cluster_addr, int v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(cluster_addr), "r"(v) : "memory");
}
// try_wait with cluster-scope acquire: data written by the other CTA of the
// pair before its release-arrive is visible after it
MOE_DEV bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
MOE_DEV bool mbar_wait_cluster(uint64_t* bar, uint32_t parity, const Abort& ab) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const unsigned long long t0 = globaltimer();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    if ((it & 63u) == 0) {
      if (ab.raised()) return false;
      if (globaltimer() - t0 > ab.limit_ns) {
        ab.raise();
        return false;
      }
    }
  }
}
// TMA load into this CTA's shared memory whose completion is counted on the
// barrier `mbar_cluster` (a shared::cluster address, normally CTA 0's)
MOE_DEV void tma_load_2d_pair(void* smem_dst, const CUtensorMap* map, uint32_t mbar_cluster,
                              int32_t x, int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(mbar_cluster), "r"(x), "r"(y)
      : "memory");
}
MOE_DEV void tmem_alloc2(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst)),
               "r"(ncols)
               : "memory");
}
MOE_DEV void tmem_relinquish2() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
MOE_DEV void tmem_dealloc2(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
MOE_DEV void umma2_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// arrive on the barrier at this shared offset in both CTAs of the pair once
// every MMA issued so far has completed
MOE_DEV void umma2_commit_both(const uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(smem_u32(bar)),
      "h"(static_cast<uint16_t>(0x3))
      : "memory");
}
MOE_DEV void umma2_commit_local(const uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

MOE_DEV void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// 32 lanes x 32 columns of 32-bit: thread i of the warp gets row (lane base + i),
// columns [col, col + 32).
MOE_DEV void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
MOE_DEV void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

// Shared-memory matrix descriptor for a K-major operand tile written by TMA
// with 128-byte swizzle: rows of 64 bf16 (128 B), 8-row groups 1024 B apart.
// `saddr` must be 1024-byte aligned (base offset 0).
MOE_DEV uint64_t smem_desc_k_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);  // start address, bits 0-13
  d |= static_cast<uint64_t>(1) << 16;                    // leading byte offset (unused here)
  d |= static_cast<uint64_t>(1024 >> 4) << 32;            // stride byte offset: 8 rows
  d |= static_cast<uint64_t>(1) << 46;                    // descriptor version (sm_100)
  d |= static_cast<uint64_t>(2) << 61;                    // layout: 128-byte swizzle
  return d;
}

// Instruction descriptor: kind::f16 with bf16 A/B, fp32 D, both K-major, M x N.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N) {
  return (1u << 4)                                   // D format: f32
         | (1u << 7)                                 // A format: bf16
         | (1u << 10)                                // B format: bf16
         | (static_cast<uint32_t>(N >> 3) << 17)     // N / 8
         | (static_cast<uint32_t>(M >> 4) << 24);    // M / 16
}


// GEGLU hidden unit from its gate and linear accumulators (GEMM-1 columns 2i
// and 2i + 1): GELU(g) * l with GELU(a) = a * Phi(a) = a (1 + erf(a / sqrt 2)) / 2.
MOE_DEV float geglu(float g, float l) {
  return 0.5f * g * (1.0f + erff(g * 0.70710678118654752f)) * l;
}
// 32 GEMM-1 accumulator columns (16 gate / linear pairs) -> 16 bf16 hidden
// units stored at dst (32 bytes, 16-byte aligned).
MOE_DEV void store_geglu16(const uint32_t (&r)[32], __nv_bfloat16* dst) {
  uint32_t packed[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float h0 = geglu(__uint_as_float(r[4 * i]), __uint_as_float(r[4 * i + 1]));
    const float h1 = geglu(__uint_as_float(r[4 * i + 2]), __uint_as_float(r[4 * i + 3]));
    __nv_bfloat162 h = __floats2bfloat162_rn(h0, h1);
    packed[i] = *reinterpret_cast<uint32_t*>(&h);
  }
  uint4* d = reinterpret_cast<uint4*>(dst);
  d[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
  d[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
}

}  // namespace dev
}  // namespace moe
