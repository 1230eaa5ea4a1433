// Grouped "TN" GEMM on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
//   out[g, m, n] = epilogue( sum_k A[g, m, k] * B[g, n, k] )
//
// for every group g (an expert, or the single router group), m < rows[g]
// (read on the device, e.g. the kept-token count of an expert) and n < N.
// Both operands are K-major bf16; accumulation is fp32 in tensor memory.
// It computes the router logits of moe_router (Switch notes sec. 2.1
// h = W_r x, fp32 per sec. 2.4: x Wr^T + bias) and the expert FFN of layers
// whose capacity lies between the ranges of the fused FFN kernels (two
// grouped launches).  The router with the gate and top-k in its epilogue is
// router_pair.cu.
//
// Design: one persistent CTA per SM walks a static list of 128 x BN output
// tiles ordered (group, n-block, m-block) so that the m-blocks sharing a
// weight tile run at the same time and the weight tile is fetched from HBM
// once.  Warp 0 issues TMA loads into a STAGES-deep ring of 128-byte-
// swizzled shared-memory tiles; warp 1 issues tcgen05.mma (M=128, N=BN,
// K=16) into one of two TMEM accumulators; warps 2-5 drain the other
// accumulator (tcgen05.ld), apply the epilogue and store, so the epilogue of
// tile i overlaps the main loop of tile i+1.  Every wait is bounded.
#include <cuda.h>

#include <climits>

#include "moe_internal.cuh"

namespace moe {
namespace {

// EPI_GLU_BF16: GEMM 1 of a GEGLU expert; accumulator columns 2i, 2i + 1 are
// hidden unit i's gate and linear parts, out gets GELU(gate) * linear.
enum EpiKind { EPI_RELU_BF16 = 0, EPI_BF16 = 1, EPI_F32_BIAS = 2, EPI_GLU_BF16 = 4 };

constexpr int kBM = 128;          // rows per tile (MMA M)
constexpr int kBK = 64;           // K per stage: one 128-byte swizzle row of bf16
constexpr int kUmmaK = 16;        // K per tcgen05.mma (kind::f16)
constexpr int kThreads = 192;     // 6 warps
constexpr int kMaxGroups = 256;

struct GemmParams {
  int32_t num_groups;
  int32_t a_group_rows;        // row stride between groups in A and out (C; 0 = one group)
  const int32_t* group_rows;   // device [num_groups] row counts, or null -> fixed_rows
  int32_t fixed_rows;
  int32_t max_rows;            // rows per group are clamped to [0, max_rows]
  int32_t N;                   // output columns
  int32_t b_group_rows;        // row stride between groups in B (N for FFN, 0 for router)
  int32_t K;
  void* out;                   // row-major, out_ld elements per row
  int64_t out_ld;
  const float* bias;           // EPI_F32_BIAS, nullable
  const int32_t* scatter_tok;  // EPI_BF16, top-1 layers: row -> token map, or null
  const float* scatter_gate;   //   gate per token
  __nv_bfloat16* scatter_y;    //   y [T, out_ld] written instead of out
  int32_t* status;             // nullable; also the call's give-up signal
  uint64_t wait_ns;            // limit of every bounded wait
};

template <int BN>
struct Cfg {
  static constexpr int kABytes = kBM * kBK * 2;  // 16 KB
  static constexpr int kBBytes = BN * kBK * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kStages = (200 * 1024) / kStageBytes > 8 ? 8 : (200 * 1024) / kStageBytes;
  static constexpr int kTmemCols = (2 * BN <= 32) ? 32 : (2 * BN <= 64) ? 64 : (2 * BN <= 128) ? 128
                                   : (2 * BN <= 256) ? 256 : 512;
  static constexpr int kAccStride = kTmemCols / 2;
  static constexpr int kSmemBytes = 1024 + kStages * kStageBytes;
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N");
  static_assert(kBBytes % 1024 == 0, "B stage alignment");
};

struct TileCoord {
  int g, m_blk, n_blk;
};

__device__ __forceinline__ TileCoord tile_of(int t, const int* prefix, const int* mblk, int G,
                                             int n_blocks) {
  int lo = 0, hi = G - 1;  // last g with prefix[g] <= t
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (prefix[mid] <= t) lo = mid; else hi = mid - 1;
  }
  int local = t - prefix[lo];
  TileCoord c;
  c.g = lo;
  c.n_blk = local / mblk[lo];
  c.m_blk = local - c.n_blk * mblk[lo];
  (void)n_blocks;
  return c;
}

template <int BN, int EPI>
__global__ void __launch_bounds__(kThreads, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
               GemmParams p) {
  using C = Cfg<BN>;
  constexpr int S = C::kStages;
  constexpr uint32_t kIdesc = dev::idesc_bf16_f32(kBM, BN);

  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t full_bar[S], empty_bar[S], tfull_bar[2], tempty_bar[2], done_bar;
  __shared__ uint32_t s_tmem_base;
  __shared__ int s_rows[kMaxGroups], s_mblk[kMaxGroups], s_prefix[kMaxGroups + 1];
  __shared__ volatile int s_abort;

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* smA = smem;
  uint8_t* smB = smem + S * C::kABytes;

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int G = p.num_groups;
  const int n_blocks = (p.N + BN - 1) / BN;
  const int num_kb = p.K / kBK;

  // ---- set-up: barriers and TMEM (no global memory), then per-group tile counts ----
  dev::pdl_trigger();
  if (tid == 0) {
    s_abort = 0;
    for (int s = 0; s < S; ++s) {
      dev::mbar_init(&full_bar[s], 1);
      dev::mbar_init(&empty_bar[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      dev::mbar_init(&tfull_bar[a], 1);
      dev::mbar_init(&tempty_bar[a], 128);
    }
    dev::mbar_init(&done_bar, 1);
    dev::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    dev::tma_prefetch_desc(&tmA);
    dev::tma_prefetch_desc(&tmB);
  }
  dev::pdl_wait();  // the previous kernel's outputs (row counts, x) are visible from here
  if (warp == 1) {  // TMEM only after the previous kernel has finished (see pdl_wait)
    dev::tmem_alloc(&s_tmem_base, C::kTmemCols);
    dev::tmem_relinquish();
  }
  for (int g = tid; g < G; g += kThreads) {
    int r = p.group_rows ? p.group_rows[g] : p.fixed_rows;
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
  dev::tc_fence_after();
  const uint32_t tmem_base = s_tmem_base;
  const int total_tiles = s_prefix[G];
  const dev::Abort ab{&s_abort, p.status, p.wait_ns};

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      long long issued = 0;
      for (int t = blockIdx.x; t < total_tiles && !ab.raised_here(); t += gridDim.x) {
        TileCoord tc = tile_of(t, s_prefix, s_mblk, G, n_blocks);
        const int a_row = tc.g * p.a_group_rows + tc.m_blk * kBM;
        const int b_row = tc.g * p.b_group_rows + tc.n_blk * BN;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!dev::mbar_wait(&empty_bar[stage], phase ^ 1u, ab)) break;
          dev::mbar_arrive_expect_tx(&full_bar[stage], C::kStageBytes);
          dev::tma_load_2d(smA + stage * C::kABytes, &tmA, &full_bar[stage], kb * kBK, a_row);
          dev::tma_load_2d(smB + stage * C::kBBytes, &tmB, &full_bar[stage], kb * kBK, b_row);
          ++issued;
          if (++stage == S) { stage = 0; phase ^= 1u; }
        }
      }
      // Make sure no bulk copy is still landing in shared memory when the CTA exits.
      const unsigned long long deadline = dev::globaltimer() + p.wait_ns;
      for (int s = 0; s < S; ++s) {
        if (issued > s) {
          long long last_fill = (issued - 1 - s) / S;
          dev::mbar_wait_drain(&full_bar[s], static_cast<uint32_t>(last_fill & 1), ab, deadline);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool any = false;
      for (int t = blockIdx.x; t < total_tiles && !ab.raised_here(); t += gridDim.x) {
        if (!dev::mbar_wait(&tempty_bar[acc], acc_phase ^ 1u, ab)) break;
        dev::tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * C::kAccStride);
        bool ok = true;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!dev::mbar_wait(&full_bar[stage], phase, ab)) { ok = false; break; }
          dev::tc_fence_after();
          const uint64_t adesc = dev::smem_desc_k_sw128(dev::smem_u32(smA + stage * C::kABytes));
          const uint64_t bdesc = dev::smem_desc_k_sw128(dev::smem_u32(smB + stage * C::kBBytes));
#pragma unroll
          for (int kk = 0; kk < kBK / kUmmaK; ++kk) {
            // advance the start address by kk * 16 elements * 2 bytes = 32 B (>> 4 = 2)
            dev::umma_bf16(d_tmem, adesc + 2ull * kk, bdesc + 2ull * kk, kIdesc,
                           (kb > 0 || kk > 0) ? 1u : 0u);
          }
          dev::umma_commit(&empty_bar[stage]);  // frees the smem stage once these MMAs finish
          any = true;
          if (++stage == S) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        dev::umma_commit(&tfull_bar[acc]);  // accumulator ready for the epilogue
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      if (any) {
        // every MMA issued by this thread has completed before TMEM is released
        dev::umma_commit(&done_bar);
        dev::mbar_wait_drain(&done_bar, 0, ab, dev::globaltimer() + p.wait_ns);
      }
    }
  } else {
    // ---------------- epilogue: warps 2..5 ----------------
    const int q = warp & 3;  // TMEM lane quarter this warp may read
    const int row_local = q * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = blockIdx.x; t < total_tiles; t += gridDim.x) {
      TileCoord tc = tile_of(t, s_prefix, s_mblk, G, n_blocks);
      // lane 0 waits; the result is broadcast so the warp stays converged for
      // the .sync.aligned tcgen05.ld below
      int ok = 0;
      if (lane == 0) ok = dev::mbar_wait(&tfull_bar[acc], acc_phase, ab) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      dev::tc_fence_after();
      const int rows_valid = s_rows[tc.g] - tc.m_blk * kBM;
      const bool row_ok = row_local < rows_valid;
      const int64_t grow = static_cast<int64_t>(tc.g) * p.a_group_rows + tc.m_blk * kBM + row_local;
      const int n0 = tc.n_blk * BN;
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                             static_cast<uint32_t>(acc * C::kAccStride);
      if constexpr (EPI == EPI_F32_BIAS) {
        float* out = static_cast<float*>(p.out) + grow * p.out_ld;
#pragma unroll 1
        for (int c = 0; c < BN / 16; ++c) {
          uint32_t r[16];
          dev::tmem_ld_32x32b_x16(tbase + c * 16, r);
          dev::tmem_wait_ld();
          const int n = n0 + c * 16;
          if (row_ok && n < p.N) {
            if (n + 16 <= p.N && (p.out_ld & 3) == 0) {
              float v[16];
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                v[i] = __uint_as_float(r[i]);
                if (p.bias) v[i] += __ldg(p.bias + n + i);
              }
              float4* dst = reinterpret_cast<float4*>(out + n);
#pragma unroll
              for (int i = 0; i < 4; ++i)
                dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
            } else {  // ragged last columns or rows not 16-byte aligned
#pragma unroll
              for (int i = 0; i < 16; ++i)
                if (n + i < p.N) out[n + i] = __uint_as_float(r[i]) + (p.bias ? __ldg(p.bias + n + i) : 0.f);
            }
          }
        }
      } else {
        __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out) + grow * p.out_ld;
        float scale = 1.f;
        if (EPI == EPI_BF16 && p.scatter_y && row_ok) {
          // top-1 combine: y[t] = gate_t * row, written in token order
          const int tok = __ldg(p.scatter_tok + grow);
          scale = __ldg(p.scatter_gate + tok);
          out = p.scatter_y + static_cast<int64_t>(tok) * p.out_ld;
        }
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t r[32];
          dev::tmem_ld_32x32b_x32(tbase + c * 32, r);
          dev::tmem_wait_ld();
          const int n = n0 + c * 32;
          if (EPI == EPI_GLU_BF16) {
            if (row_ok && n < p.N) dev::store_geglu16(r, out + n / 2);
          } else if (row_ok && n < p.N) {
            uint32_t packed[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              float a = __uint_as_float(r[2 * i]) * scale;
              float b = __uint_as_float(r[2 * i + 1]) * scale;
              if (EPI == EPI_RELU_BF16) { a = fmaxf(a, 0.f); b = fmaxf(b, 0.f); }
              __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
              packed[i] = *reinterpret_cast<uint32_t*>(&h);
            }
            uint4* dst = reinterpret_cast<uint4*>(out + n);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              dst[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
          }
        }
      }
      dev::tc_fence_before();
      dev::mbar_arrive(&tempty_bar[acc]);
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
  }

  dev::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    dev::tc_fence_after();
    dev::tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

// ---- host side ----------------------------------------------------------------

template <int BN, int EPI>
int32_t launch_gemm(const void* A, uint64_t a_rows, const void* B, uint64_t b_rows,
                    const GemmParams& p, int64_t max_tiles, cudaStream_t s) {
  using C = Cfg<BN>;
  if (max_tiles <= 0) return MOE_OK;
  CUtensorMap ta, tb;
  int32_t rc = make_tmap_bf16(&ta, A, a_rows, static_cast<uint64_t>(p.K), kBM);
  if (rc != MOE_OK) return rc;
  rc = make_tmap_bf16(&tb, B, b_rows, static_cast<uint64_t>(p.K), BN);
  if (rc != MOE_OK) return rc;
  auto kern = gemm_tc_kernel<BN, EPI>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) !=
      cudaSuccess)
    return check_launch("cudaFuncSetAttribute(gemm_tc_kernel)");
  int grid = static_cast<int>(max_tiles < num_sms() ? max_tiles : num_sms());
  launch_pdl(kern, dim3(grid), dim3(kThreads), C::kSmemBytes, s, ta, tb, p);
  return check_launch("gemm_tc_kernel");
}

}  // namespace

// Expert FFN as two grouped launches (GEMM 1 then GEMM 2), used when experts
// span several 128-row blocks: the static tile order keeps the CTAs that
// share a weight tile in lockstep, so its k-slices are served once from L2.
int32_t launch_ffn_two_pass(const moe_config& c, const void* xe, const void* W1, const void* W2,
                            const int32_t* kept_cnt, void* H, void* ye, int32_t* status,
                            cudaStream_t s, const Top1Out* top1) {
  const int64_t E = c.E, C = c.capacity, d = c.d_model, f = c.d_ff;
  if (E == 0 || C == 0) return MOE_OK;
  const int64_t mblk_max = (C + kBM - 1) / kBM;
  GemmParams p{};
  p.num_groups = c.E;
  p.a_group_rows = c.capacity;
  p.group_rows = kept_cnt;
  p.fixed_rows = 0;
  p.max_rows = c.capacity;
  p.status = status;
  p.wait_ns = wait_limit_ns();
  p.bias = nullptr;
  // GEMM 1: [E*C, d] x [E*f, d]^T -> H [E*C, f], ReLU; GEGLU: W1 has 2f rows
  // per expert and each pair of accumulator columns gives one unit of H
  const bool glu = c.expert == MOE_EXPERT_GEGLU;
  const int64_t n1 = glu ? 2 * f : f;
  p.N = static_cast<int32_t>(n1);
  p.b_group_rows = static_cast<int32_t>(n1);
  p.K = c.d_model;
  p.out = H;
  p.out_ld = f;
  const int64_t t1 = E * mblk_max * ((n1 + 255) / 256);
  int32_t rc = glu ? launch_gemm<256, EPI_GLU_BF16>(xe, E * C, W1, E * n1, p, t1, s)
                   : launch_gemm<256, EPI_RELU_BF16>(xe, E * C, W1, E * n1, p, t1, s);
  if (rc != MOE_OK) return rc;
  // GEMM 2: [E*C, f] x [E*d, f]^T -> ye [E*C, d]
  p.N = c.d_model;
  p.b_group_rows = c.d_model;
  p.K = c.d_ff;
  p.out = ye;
  p.out_ld = d;
  if (top1) {
    p.scatter_tok = top1->tok_of_row;
    p.scatter_gate = top1->gate;
    p.scatter_y = static_cast<__nv_bfloat16*>(top1->y);
  }
  return launch_gemm<256, EPI_BF16>(H, E * C, W2, E * d, p, E * mblk_max * ((d + 255) / 256), s);
}

// logits [T, E] fp32 = x [T, d] . Wr [E, d]^T + bias
int32_t launch_router_tc(const moe_config& c, const void* x, const void* Wr, const float* bias,
                         float* logits, int32_t* status, cudaStream_t s) {
  if (c.T == 0) return MOE_OK;
  GemmParams p{};
  p.num_groups = 1;
  p.a_group_rows = 0;
  p.group_rows = nullptr;
  p.fixed_rows = static_cast<int32_t>(c.T);
  p.max_rows = static_cast<int32_t>(c.T);
  p.N = c.E;
  p.b_group_rows = 0;
  p.K = c.d_model;
  p.out = logits;
  p.out_ld = c.E;
  p.bias = bias;
  p.status = status;
  p.wait_ns = wait_limit_ns();
  const int64_t tiles = (c.T + kBM - 1) / kBM;
  const uint64_t T = static_cast<uint64_t>(c.T), E = static_cast<uint64_t>(c.E);
  if (c.E <= 32) return launch_gemm<32, EPI_F32_BIAS>(x, T, Wr, E, p, tiles, s);
  if (c.E <= 64) return launch_gemm<64, EPI_F32_BIAS>(x, T, Wr, E, p, tiles, s);
  if (c.E <= 128) return launch_gemm<128, EPI_F32_BIAS>(x, T, Wr, E, p, tiles, s);
  return launch_gemm<256, EPI_F32_BIAS>(x, T, Wr, E, p, tiles, s);
}

}  // namespace moe
