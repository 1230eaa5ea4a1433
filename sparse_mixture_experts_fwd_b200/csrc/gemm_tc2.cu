// Grouped expert GEMM on SM pairs (tcgen05 cta_group::2), for layers whose
// experts hold many rows (the tensor-core-bound case).
//
//   out[e, m, n] = epilogue( sum_k A[e, m, k] * B[e, n, k] ),  m < rows[e]
//
// A cluster of two CTAs (one per SM) computes a 256 x 256 output tile with
// tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 16): CTA r holds rows
// [128r, 128r + 128) of the A tile and rows [128r, 128r + 128) of the B tile
// (N half) in its own shared memory, and its TMEM holds its 128 output rows
// x 256 columns.  Per SM this needs 32 KB of operands per 64-deep k-block
// instead of 48 KB for a 128 x 256 single-CTA tile, so the operand feed, which
// limits the single-CTA kernel, carries a third less and 6 stages fit.
//
// Roles: in each CTA warp 0 lane 0 loads its halves with TMA; the loads of
// both CTAs complete on CTA 0's "full" barrier, which CTA 0 arms with the
// pair's byte count.  CTA 0's warp 1 lane 0 issues the MMAs and commits them
// with one tcgen05.commit that arrives on both CTAs' "empty" (stage free) and
// "tfull" (accumulator ready) barriers.  Warps 2-5 of each CTA drain their own
// TMEM and arrive on CTA 0's "tempty" barrier (remotely from CTA 1).  Every
// wait is bounded; a cluster barrier brackets the kernel so neither CTA frees
// TMEM or exits while the other still uses it.  Each CTA's TMA loads fill only
// its own shared memory.
#include <cuda.h>

#include <algorithm>

#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int kHalf = 128;          // rows of A and of B per CTA
constexpr int kBM = 256, kBN = 256, kBK = 64, kUmmaK = 16;
constexpr int kThreads = 192;
constexpr int kStages = 6;
constexpr int kABytes = kHalf * kBK * 2;  // 16 KB
constexpr int kBBytes = kHalf * kBK * 2;  // 16 KB
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kTmemCols = 512;
constexpr int kAccStride = 256;
constexpr int kMaxGroups = 256;
constexpr int kSmemBytes = 1024 + kStages * kStageBytes;
constexpr uint32_t kIdesc = dev::idesc_bf16_f32(kBM, kBN);

// EPI2_GLU_BF16: GEMM 1 of a GEGLU expert (column pairs -> GELU(gate) * linear)
enum Epi2 { EPI2_RELU_BF16 = 0, EPI2_BF16 = 1, EPI2_GLU_BF16 = 2 };

struct Gemm2Params {
  int32_t num_groups;
  int32_t a_group_rows;  // row stride between groups in A and out
  const int32_t* group_rows;
  int32_t max_rows;
  int32_t N;
  int32_t b_group_rows;
  int32_t K;
  __nv_bfloat16* out;
  int64_t out_ld;
  int32_t* status;             // nullable; also the call's give-up signal
  uint64_t wait_ns;            // limit of every bounded wait
  const int32_t* scatter_tok;  // EPI2_BF16, top-1 layers: row -> token map, or null
  const float* scatter_gate;   //   gate per token
  __nv_bfloat16* scatter_y;    //   y [T, out_ld] written instead of out
};

using dev::cluster_sync;
using dev::cta_rank;
using dev::mapa;
using dev::mbar_arrive_cluster;
using dev::tma_load_2d_pair;
using dev::tmem_alloc2;
using dev::tmem_dealloc2;
using dev::tmem_relinquish2;
using dev::umma2_commit_both;
using dev::umma2_commit_local;

struct TileCoord {
  int g, m, n;  // m: 256-row block
};

MOE_DEV TileCoord tile_of(int t, const int* prefix, const int* mblk, int G) {
  int lo = 0, hi = G - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (prefix[mid] <= t) lo = mid; else hi = mid - 1;
  }
  const int local = t - prefix[lo];
  TileCoord c;
  c.g = lo;
  c.n = local / mblk[lo];
  c.m = local - c.n * mblk[lo];
  return c;
}

template <int EPI>
__global__ void __launch_bounds__(kThreads, 1)
gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 Gemm2Params p) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t full_bar[kStages], empty_bar[kStages], tfull_bar[2], tempty_bar[2], done_bar;
  __shared__ uint32_t s_tmem_base;
  __shared__ int s_rows[kMaxGroups], s_mblk[kMaxGroups], s_prefix[kMaxGroups + 1];
  __shared__ volatile int s_abort;

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* smA = smem;
  uint8_t* smB = smem + kStages * kABytes;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cta_rank();
  const int cluster = blockIdx.x >> 1;
  const int n_clusters = gridDim.x >> 1;
  const int G = p.num_groups;
  const int n_blocks = (p.N + kBN - 1) / kBN;
  const int num_kb = p.K / kBK;

  dev::pdl_trigger();
  if (tid == 0) {
    s_abort = 0;
    for (int s = 0; s < kStages; ++s) {
      dev::mbar_init(&full_bar[s], 1);
      dev::mbar_init(&empty_bar[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      dev::mbar_init(&tfull_bar[a], 1);
      dev::mbar_init(&tempty_bar[a], 2 * 128);  // epilogue threads of both CTAs (used in CTA 0)
    }
    dev::mbar_init(&done_bar, 1);
    dev::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    dev::tma_prefetch_desc(&tmA);
    dev::tma_prefetch_desc(&tmB);
  }
  dev::pdl_wait();
  if (warp == 1) {  // TMEM only after the previous kernel has finished (see pdl_wait)
    tmem_alloc2(&s_tmem_base, kTmemCols);
    tmem_relinquish2();
  }
  for (int g = tid; g < G; g += kThreads) {
    int r = p.group_rows[g];
    r = r < 0 ? 0 : (r > p.max_rows ? p.max_rows : r);
    s_rows[g] = r;
    s_mblk[g] = (r + kBM - 1) / kBM;
  }
  __syncthreads();
  if (tid == 0) {
    int acc = 0;
    for (int g = 0; g < G; ++g) {
      s_prefix[g] = acc;
      acc += s_mblk[g] * n_blocks;
    }
    s_prefix[G] = acc;
  }
  dev::tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers are initialised and TMEM allocated
  dev::tc_fence_after();
  const uint32_t tmem_base = s_tmem_base;
  const int total = s_prefix[G];
  const dev::Abort ab{&s_abort, p.status, p.wait_ns};

  if (warp == 0) {
    // ---------------- TMA producer (both CTAs) ----------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      long long issued = 0;
      for (int t = cluster; t < total && !ab.raised_here(); t += n_clusters) {
        const TileCoord tc = tile_of(t, s_prefix, s_mblk, G);
        const int a_row = tc.g * p.a_group_rows + tc.m * kBM + static_cast<int>(rank) * kHalf;
        const int b_row = tc.g * p.b_group_rows + tc.n * kBN + static_cast<int>(rank) * kHalf;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!dev::mbar_wait(&empty_bar[stage], phase ^ 1u, ab)) break;
          if (rank == 0) dev::mbar_arrive_expect_tx(&full_bar[stage], 2 * kStageBytes);
          const uint32_t full0 = mapa(&full_bar[stage], 0);  // CTA 0's barrier for this stage
          tma_load_2d_pair(smA + stage * kABytes, &tmA, full0, kb * kBK, a_row);
          tma_load_2d_pair(smB + stage * kBBytes, &tmB, full0, kb * kBK, b_row);
          ++issued;
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
      }
      if (rank == 0) {
        // the pair's copies have all landed once CTA 0's full barriers complete
        const unsigned long long deadline = dev::globaltimer() + p.wait_ns;
        for (int s = 0; s < kStages; ++s) {
          if (issued > s) {
            const long long last_fill = (issued - 1 - s) / kStages;
            dev::mbar_wait_drain(&full_bar[s], static_cast<uint32_t>(last_fill & 1), ab, deadline);
          }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (CTA 0 only) ----------------
    if (lane == 0 && rank == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool any = false;
      for (int t = cluster; t < total && !ab.raised_here(); t += n_clusters) {
        if (!dev::mbar_wait(&tempty_bar[acc], acc_phase ^ 1u, ab)) break;
        dev::tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kAccStride);
        bool ok = true;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!dev::mbar_wait(&full_bar[stage], phase, ab)) { ok = false; break; }
          dev::tc_fence_after();
          const uint64_t adesc = dev::smem_desc_k_sw128(dev::smem_u32(smA + stage * kABytes));
          const uint64_t bdesc = dev::smem_desc_k_sw128(dev::smem_u32(smB + stage * kBBytes));
#pragma unroll
          for (int kk = 0; kk < kBK / kUmmaK; ++kk)
            dev::umma2_bf16(d_tmem, adesc + 2ull * kk, bdesc + 2ull * kk, kIdesc,
                            (kb > 0 || kk > 0) ? 1u : 0u);
          umma2_commit_both(&empty_bar[stage]);
          any = true;
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma2_commit_both(&tfull_bar[acc]);
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      if (any) {
        umma2_commit_local(&done_bar);
        dev::mbar_wait_drain(&done_bar, 0, ab, dev::globaltimer() + p.wait_ns);
      }
    }
  } else {
    // ---------------- epilogue: warps 2..5 of both CTAs ----------------
    const int q = warp & 3;
    const int row_local = q * 32 + lane;
    const uint32_t tempty_c0 = mapa(&tempty_bar[0], 0);
    const uint32_t tempty_c1 = mapa(&tempty_bar[1], 0);
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = cluster; t < total; t += n_clusters) {
      const TileCoord tc = tile_of(t, s_prefix, s_mblk, G);
      int ok = 0;
      if (lane == 0) ok = dev::mbar_wait(&tfull_bar[acc], acc_phase, ab) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      dev::tc_fence_after();
      const int row_in_group = tc.m * kBM + static_cast<int>(rank) * kHalf + row_local;
      const bool row_ok = row_in_group < s_rows[tc.g];
      const int64_t grow = static_cast<int64_t>(tc.g) * p.a_group_rows + row_in_group;
      __nv_bfloat16* out = p.out + grow * p.out_ld;
      float scale = 1.f;
      if (EPI == EPI2_BF16 && p.scatter_y && row_ok) {
        // top-1 combine: y[t] = gate_t * row, written in token order
        const int tok = __ldg(p.scatter_tok + grow);
        scale = __ldg(p.scatter_gate + tok);
        out = p.scatter_y + static_cast<int64_t>(tok) * p.out_ld;
      }
      const int n0 = tc.n * kBN;
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                             static_cast<uint32_t>(acc * kAccStride);
#pragma unroll 1
      for (int c = 0; c < kBN / 32; ++c) {
        uint32_t r[32];
        dev::tmem_ld_32x32b_x32(tbase + c * 32, r);
        dev::tmem_wait_ld();
        const int n = n0 + c * 32;
        if (EPI == EPI2_GLU_BF16) {
          if (row_ok && n < p.N) dev::store_geglu16(r, out + n / 2);
        } else if (row_ok && n < p.N) {
          uint32_t packed[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float a = __uint_as_float(r[2 * i]) * scale;
            float b = __uint_as_float(r[2 * i + 1]) * scale;
            if (EPI == EPI2_RELU_BF16) { a = fmaxf(a, 0.f); b = fmaxf(b, 0.f); }
            __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
            packed[i] = *reinterpret_cast<uint32_t*>(&h);
          }
          uint4* dst = reinterpret_cast<uint4*>(out + n);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            dst[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
        }
      }
      dev::tc_fence_before();
      mbar_arrive_cluster(acc == 0 ? tempty_c0 : tempty_c1);  // CTA 0's accumulator-free barrier
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
  }

  dev::tc_fence_before();
  __syncthreads();
  cluster_sync();  // no CTA frees TMEM or exits while its partner's MMAs or copies may run
  if (warp == 1) {
    __syncwarp();
    dev::tc_fence_after();
    tmem_dealloc2(tmem_base, kTmemCols);
  }
}


template <int EPI>
int32_t launch_pair(const void* A, uint64_t a_rows, const void* B, uint64_t b_rows,
                    const Gemm2Params& p, int64_t max_tiles, cudaStream_t s) {
  if (max_tiles <= 0) return MOE_OK;
  CUtensorMap ta, tb;
  int32_t rc = make_tmap_bf16(&ta, A, a_rows, static_cast<uint64_t>(p.K), kHalf);
  if (rc != MOE_OK) return rc;
  rc = make_tmap_bf16(&tb, B, b_rows, static_cast<uint64_t>(p.K), kHalf);
  if (rc != MOE_OK) return rc;
  auto kern = gemm_pair_kernel<EPI>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) !=
      cudaSuccess)
    return check_launch("cudaFuncSetAttribute(gemm_pair_kernel)");
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(num_sms() & ~1));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;  // cluster shape only, for the occupancy query
  // the static tile schedule assumes every cluster is resident at once
  int resident = 0;
  if (cudaOccupancyMaxActiveClusters(&resident, kern, &cfg) != cudaSuccess || resident < 1)
    return check_launch("cudaOccupancyMaxActiveClusters(gemm_pair_kernel)");
  const int64_t clusters = std::min<int64_t>(resident, max_tiles);
  cfg.gridDim = dim3(static_cast<unsigned>(2 * clusters));
  cfg.numAttrs = 2;
  cudaLaunchKernelEx(&cfg, kern, ta, tb, p);
  return check_launch("gemm_pair_kernel");
}

}  // namespace

// H = ReLU(xe W1^T), ye = H W2^T on SM pairs, 256 x 256 tiles.
int32_t launch_ffn_pairs(const moe_config& c, const void* xe, const void* W1, const void* W2,
                         const int32_t* kept_cnt, void* H, void* ye, int32_t* status,
                         cudaStream_t s, const Top1Out* top1) {
  const int64_t E = c.E, C = c.capacity, d = c.d_model, f = c.d_ff;
  if (E == 0 || C == 0) return MOE_OK;
  const int64_t mblk_max = (C + kBM - 1) / kBM;
  Gemm2Params p{};
  p.num_groups = c.E;
  p.a_group_rows = c.capacity;
  p.group_rows = kept_cnt;
  p.max_rows = c.capacity;
  p.status = status;
  p.wait_ns = wait_limit_ns();
  // GEGLU: W1 has 2f rows per expert, each accumulator column pair one unit of H
  const bool glu = c.expert == MOE_EXPERT_GEGLU;
  const int64_t n1 = glu ? 2 * f : f;
  p.N = static_cast<int32_t>(n1);
  p.b_group_rows = static_cast<int32_t>(n1);
  p.K = c.d_model;
  p.out = static_cast<__nv_bfloat16*>(H);
  p.out_ld = f;
  const int64_t t1 = E * mblk_max * ((n1 + kBN - 1) / kBN);
  int32_t rc = glu ? launch_pair<EPI2_GLU_BF16>(xe, E * C, W1, E * n1, p, t1, s)
                   : launch_pair<EPI2_RELU_BF16>(xe, E * C, W1, E * n1, p, t1, s);
  if (rc != MOE_OK) return rc;
  p.N = c.d_model;
  p.b_group_rows = c.d_model;
  p.K = c.d_ff;
  p.out = static_cast<__nv_bfloat16*>(ye);
  p.out_ld = d;
  if (top1) {
    p.scatter_tok = top1->tok_of_row;
    p.scatter_gate = top1->gate;
    p.scatter_y = static_cast<__nv_bfloat16*>(top1->y);
  }
  return launch_pair<EPI2_BF16>(H, E * C, W2, E * d, p, E * mblk_max * ((d + kBN - 1) / kBN), s);
}

}  // namespace moe
