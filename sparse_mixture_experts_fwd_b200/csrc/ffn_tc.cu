// Expert FFN for bf16 layers (Switch notes sec. 2.1, the experts E_i):
//   H[e]  = round(ReLU(xe[e] W1[e]^T))     GEMM 1, K = d_model
//   ye[e] = round(H[e] W2[e]^T)            GEMM 2, K = d_ff
// over each expert's kept rows, as ONE persistent tcgen05 kernel.
//
// Tiles are 128 rows x 256 columns.  They form one sequence of "units":
// unit u holds the GEMM-1 tiles of expert u followed by the GEMM-2 tiles of
// expert u - L (L = lag), tiles of one expert ordered (n-block, m-block) so
// that the m-blocks sharing a weight tile run side by side and each weight
// byte leaves HBM once.  CTAs (one per SM) grab the next tile from a global
// counter, so the load balances to within one tile and GEMM 2 fills the SMs
// while GEMM 1 of later experts is still running — no tail between the two
// GEMMs and no second launch.  A GEMM-2 tile of expert e needs all of H[e]:
// every epilogue warp that finished its rows of a GEMM-1 tile increments
// done1[e] (release) and the producer of
// a GEMM-2 tile waits (acquire, bounded) until done1[e] counts all of them.
// The lag L is chosen so that this wait is normally already satisfied.
//
// Roles per CTA (192 threads): warp 0 lane 0 grabs tiles, publishes them in a
// shared-memory ring and issues TMA loads into a 4-stage operand ring; warp 1
// lane 0 issues tcgen05.mma (M=128, N=256, K=16) into one of two TMEM
// accumulators; warps 2-5 drain the other accumulator (ReLU / bf16 convert /
// store).  Every wait is bounded; on a timeout the CTA sets the status word,
// lets its copies and MMAs finish, frees TMEM and returns.
#include <cuda.h>

#include <algorithm>

#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int kBM = 128, kBN = 256, kBK = 64, kUmmaK = 16;
constexpr int kThreads = 192;
constexpr int kStages = 4;
constexpr int kRing = 8;  // tile ids in flight between the producer and the consumers
constexpr int kABytes = kBM * kBK * 2;
constexpr int kBBytes = kBN * kBK * 2;
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kTmemCols = 512;
constexpr int kAccStride = 256;
constexpr int kMaxE = 256;
constexpr int kMaxUnits = 2 * kMaxE;
constexpr int kSmemBytes = 1024 + kStages * kStageBytes;
constexpr uint32_t kIdesc = dev::idesc_bf16_f32(kBM, kBN);

struct FfnParams {
  int E, C, d, f, lag;
  int n1;                  // GEMM-1 output columns: f (ReLU) or 2f (GEGLU: gate/linear pairs)
  int glu;                 // 1: GEGLU expert
  const int32_t* kept_cnt;
  __nv_bfloat16* H;
  __nv_bfloat16* ye;
  unsigned int* tile_ctr;  // zero before launch
  unsigned int* done1;     // [E], zero before launch
  int32_t* status;         // nullable; also the call's give-up signal
  uint64_t wait_ns;        // limit of every bounded wait
  // top-1 layers: GEMM 2 writes gate * row straight to y [T, d] in token order
  // (ye untouched); null -> write ye
  const int32_t* tok_of_row;
  const float* gate;
  __nv_bfloat16* y;
};

struct Tile {
  int kind;  // 1: GEMM 1, 2: GEMM 2
  int e, m, n;
};

struct Sched {
  int E, lag, nb1, nb2;
  const int* mblk;
  const int* prefix;  // [units + 1]
  int units;

  __device__ int g1(int u) const { return u < E ? mblk[u] * nb1 : 0; }
  __device__ int g2(int u) const { return (u >= lag && u - lag < E) ? mblk[u - lag] * nb2 : 0; }

  __device__ Tile decode(int t) const {
    int lo = 0, hi = units - 1;  // last unit with prefix <= t
    while (lo < hi) {
      int mid = (lo + hi + 1) >> 1;
      if (prefix[mid] <= t) lo = mid; else hi = mid - 1;
    }
    int local = t - prefix[lo];
    Tile x;
    const int a = g1(lo);
    if (local < a) {
      x.kind = 1;
      x.e = lo;
      x.n = local / mblk[lo];
      x.m = local - x.n * mblk[lo];
    } else {
      local -= a;
      x.kind = 2;
      x.e = lo - lag;
      x.n = local / mblk[x.e];
      x.m = local - x.n * mblk[x.e];
    }
    return x;
  }
};

MOE_DEV unsigned int ld_acquire_u32(const unsigned int* p) {
  unsigned int v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
MOE_DEV void red_release_add_u32(unsigned int* p, unsigned int v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
MOE_DEV void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Bounded wait until *p has reached `need` (acquire), compared as the signed
// difference *p - need >= 0, so a counter started below zero (a caller-set
// state that no tile can complete) waits until the limit.  False on timeout /
// give-up.
MOE_DEV bool wait_count(const unsigned int* p, unsigned int need, const dev::Abort& ab) {
  if (static_cast<int>(ld_acquire_u32(p) - need) >= 0) return true;
  const unsigned long long t0 = dev::globaltimer();
  for (uint32_t it = 1;; ++it) {
    if (static_cast<int>(ld_acquire_u32(p) - need) >= 0) return true;
    if ((it & 15u) == 0) {
      if (ab.raised()) return false;
      if (dev::globaltimer() - t0 > ab.limit_ns) {
        ab.raise();
        return false;
      }
      __nanosleep(64);
    }
  }
}

__global__ void __launch_bounds__(kThreads, 1)
ffn_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW1,
              const __grid_constant__ CUtensorMap tmH, const __grid_constant__ CUtensorMap tmW2,
              FfnParams p) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t full_bar[kStages], empty_bar[kStages], tfull_bar[2], tempty_bar[2], done_bar;
  __shared__ uint64_t ring_full[kRing], ring_empty[kRing];
  __shared__ int s_ring[kRing];
  __shared__ uint32_t s_tmem_base;
  __shared__ int s_rows[kMaxE], s_mblk[kMaxE], s_prefix[kMaxUnits + 1];
  __shared__ volatile int s_abort;

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* smA = smem;
  uint8_t* smB = smem + kStages * kABytes;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int E = p.E;
  Sched sc;
  sc.E = E;
  sc.lag = p.lag;
  sc.nb1 = (p.n1 + kBN - 1) / kBN;
  sc.nb2 = (p.d + kBN - 1) / kBN;
  sc.mblk = s_mblk;
  sc.prefix = s_prefix;
  sc.units = E + p.lag;

  dev::pdl_trigger();
  if (tid == 0) {
    s_abort = 0;
    for (int s = 0; s < kStages; ++s) {
      dev::mbar_init(&full_bar[s], 1);
      dev::mbar_init(&empty_bar[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      dev::mbar_init(&tfull_bar[a], 1);
      dev::mbar_init(&tempty_bar[a], 128);
    }
    for (int r = 0; r < kRing; ++r) {
      dev::mbar_init(&ring_full[r], 1);
      dev::mbar_init(&ring_empty[r], 1 + 4);  // the MMA lane and one lane per epilogue warp
    }
    dev::mbar_init(&done_bar, 1);
    dev::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    dev::tma_prefetch_desc(&tmX);
    dev::tma_prefetch_desc(&tmW1);
    dev::tma_prefetch_desc(&tmH);
    dev::tma_prefetch_desc(&tmW2);
  }
  dev::pdl_wait();  // kept counts, xe and the zeroed counters are visible from here
  if (warp == 1) {  // TMEM only after the previous kernel has finished (see pdl_wait)
    dev::tmem_alloc(&s_tmem_base, kTmemCols);
    dev::tmem_relinquish();
  }
  for (int e = tid; e < E; e += kThreads) {
    int r = p.kept_cnt[e];
    r = r < 0 ? 0 : (r > p.C ? p.C : r);
    s_rows[e] = r;
    s_mblk[e] = (r + kBM - 1) / kBM;
  }
  __syncthreads();
  if (tid == 0) {
    int acc = 0;
    for (int u = 0; u < sc.units; ++u) {
      s_prefix[u] = acc;
      acc += sc.g1(u) + sc.g2(u);
    }
    s_prefix[sc.units] = acc;
  }
  dev::tc_fence_before();
  __syncthreads();
  dev::tc_fence_after();
  const uint32_t tmem_base = s_tmem_base;
  const int total = s_prefix[sc.units];
  const dev::Abort ab{&s_abort, p.status, p.wait_ns};

  if (warp == 0) {
    // ---------------- tile grabber + TMA producer ----------------
    if (lane == 0) {
      const uint64_t pol_w = dev::policy_evict_first();  // weights: streamed once
      const uint64_t pol_a = dev::policy_evict_last();   // activations: reread per n-block
      int slot = 0;
      uint32_t rphase = 0;
      int stage = 0;
      uint32_t phase = 0;
      long long issued = 0;
      while (!ab.raised_here()) {
        int t = static_cast<int>(atomicAdd(p.tile_ctr, 1u));
        if (t < 0 || t >= total) t = -1;  // (negative only from a counter not zeroed)
        if (!dev::mbar_wait(&ring_empty[slot], rphase ^ 1u, ab)) break;
        s_ring[slot] = t;
        dev::mbar_arrive(&ring_full[slot]);
        if (++slot == kRing) { slot = 0; rphase ^= 1u; }
        if (t < 0) break;
        const Tile x = sc.decode(t);
        const CUtensorMap* ta = x.kind == 1 ? &tmX : &tmH;
        const CUtensorMap* tb = x.kind == 1 ? &tmW1 : &tmW2;
        const int K = x.kind == 1 ? p.d : p.f;
        const int b_rows = x.kind == 1 ? p.n1 : p.d;
        if (x.kind == 2) {
          // all GEMM-1 tiles of this expert must have stored H (4 warp arrivals per tile)
          const unsigned int need = static_cast<unsigned int>(4 * s_mblk[x.e] * sc.nb1);
          if (!wait_count(p.done1 + x.e, need, ab)) break;
          fence_proxy_async_global();  // generic-proxy H stores -> async-proxy (TMA) reads
        }
        const int a_row = x.e * p.C + x.m * kBM;
        const int b_row = x.e * b_rows + x.n * kBN;
        bool ok = true;
        for (int kb = 0; kb < K / kBK; ++kb) {
          if (!dev::mbar_wait(&empty_bar[stage], phase ^ 1u, ab)) { ok = false; break; }
          dev::mbar_arrive_expect_tx(&full_bar[stage], kStageBytes);
          dev::tma_load_2d(smA + stage * kABytes, ta, &full_bar[stage], kb * kBK, a_row, pol_a);
          dev::tma_load_2d(smB + stage * kBBytes, tb, &full_bar[stage], kb * kBK, b_row, pol_w);
          ++issued;
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
      }
      const unsigned long long deadline = dev::globaltimer() + p.wait_ns;
      for (int s = 0; s < kStages; ++s) {
        if (issued > s) {
          const long long last_fill = (issued - 1 - s) / kStages;
          dev::mbar_wait_drain(&full_bar[s], static_cast<uint32_t>(last_fill & 1), ab, deadline);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      int slot = 0;
      uint32_t rphase = 0;
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool any = false;
      while (true) {
        if (!dev::mbar_wait(&ring_full[slot], rphase, ab)) break;
        const int t = s_ring[slot];
        dev::mbar_arrive(&ring_empty[slot]);
        if (++slot == kRing) { slot = 0; rphase ^= 1u; }
        if (t < 0) break;
        const Tile x = sc.decode(t);
        const int num_kb = (x.kind == 1 ? p.d : p.f) / kBK;
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
            dev::umma_bf16(d_tmem, adesc + 2ull * kk, bdesc + 2ull * kk, kIdesc,
                           (kb > 0 || kk > 0) ? 1u : 0u);
          dev::umma_commit(&empty_bar[stage]);
          any = true;
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        dev::umma_commit(&tfull_bar[acc]);
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      if (any) {
        dev::umma_commit(&done_bar);
        dev::mbar_wait_drain(&done_bar, 0, ab, dev::globaltimer() + p.wait_ns);
      }
    }
  } else {
    // ---------------- epilogue: warps 2..5 ----------------
    const int q = warp & 3;  // TMEM lane quarter this warp may read
    const int row_local = q * 32 + lane;
    int slot = 0;
    uint32_t rphase = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    while (true) {
      int t = -1, ok = 0;
      if (lane == 0) {
        ok = dev::mbar_wait(&ring_full[slot], rphase, ab) ? 1 : 0;
        if (ok) {
          t = s_ring[slot];
          dev::mbar_arrive(&ring_empty[slot]);
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      t = __shfl_sync(0xffffffffu, t, 0);
      if (!ok || t < 0) break;
      if (++slot == kRing) { slot = 0; rphase ^= 1u; }
      const Tile x = sc.decode(t);
      if (lane == 0) ok = dev::mbar_wait(&tfull_bar[acc], acc_phase, ab) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      dev::tc_fence_after();
      const int rows_valid = s_rows[x.e] - x.m * kBM;
      const bool row_ok = row_local < rows_valid;
      const int64_t grow = static_cast<int64_t>(x.e) * p.C + x.m * kBM + row_local;
      const int N = x.kind == 1 ? p.n1 : p.d;       // this GEMM's output columns
      const int ld = x.kind == 1 ? p.f : p.d;        // row stride of H / ye / y
      __nv_bfloat16* out = (x.kind == 1 ? p.H : p.ye) + grow * ld;
      float scale = 1.f;
      if (x.kind == 2 && p.y && row_ok) {
        // top-1 combine (eq. 2 with one expert): y[t] = gate_t * E(x_t), into token order
        const int tok = __ldg(p.tok_of_row + grow);
        scale = __ldg(p.gate + tok);
        out = p.y + static_cast<int64_t>(tok) * ld;
      }
      const int n0 = x.n * kBN;
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                             static_cast<uint32_t>(acc * kAccStride);
      const bool relu = x.kind == 1;
      const bool glu = x.kind == 1 && p.glu;
#pragma unroll 1
      for (int c = 0; c < kBN / 32; ++c) {
        uint32_t r[32];
        dev::tmem_ld_32x32b_x32(tbase + c * 32, r);
        dev::tmem_wait_ld();
        const int n = n0 + c * 32;
        if (glu) {
          if (row_ok && n < N) dev::store_geglu16(r, out + n / 2);
        } else if (row_ok && n < N) {
          uint32_t packed[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float a = __uint_as_float(r[2 * i]) * scale;
            float b = __uint_as_float(r[2 * i + 1]) * scale;
            if (relu) { a = fmaxf(a, 0.f); b = fmaxf(b, 0.f); }
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
      dev::mbar_arrive(&tempty_bar[acc]);
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      if (x.kind == 1) {
        // publish this warp's 32 rows of H: each thread's stores are fenced,
        // then one release increment per warp (4 per tile), so no warp ever
        // waits on another here
        fence_proxy_async_global();
        __threadfence();
        __syncwarp();
        if (lane == 0) red_release_add_u32(p.done1 + x.e, 1u);
      }
    }
  }

  dev::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    dev::tc_fence_after();
    dev::tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace

// tile counter, then one counter per (expert, chunk of at most 256 rows)
size_t ffn_sync_bytes(const moe_config& c) {
  return align256(sizeof(unsigned int) *
                  (1 + static_cast<size_t>(c.E) * static_cast<size_t>(ffn_pair_chunks(c))));
}

int32_t launch_ffn_tc(const moe_config& c, const void* xe, const void* W1, const void* W2,
                      const int32_t* kept_cnt, void* H, void* ye, void* sync, bool sync_zeroed,
                      int32_t* status, cudaStream_t s, const Top1Out* top1) {
  const int64_t E = c.E, C = c.capacity, d = c.d_model, f = c.d_ff;
  if (E == 0 || C == 0) return MOE_OK;
  if (C >= 512) {
    // Experts with hundreds of rows make the GEMMs tensor-core bound; SM
    // pairs feed each SM a third fewer operand bytes per flop than single
    // CTAs.  With a long GEMM-1 K (d_model >= 2048) both GEMMs run in one
    // launch with the tokens on the MMA's N side in 16-row steps (a ragged
    // expert wastes almost no MMA rows, H stays in L2); with a short one the
    // transposed epilogue of that kernel costs more than it saves, and two
    // launches with the tokens as M (256-row blocks) measured faster.
    if (d >= 2048)
      return launch_ffn_pair_fused(c, xe, W1, W2, kept_cnt, H, ye, sync, sync_zeroed, status,
                                   s, top1);
    return launch_ffn_pairs(c, xe, W1, W2, kept_cnt, H, ye, status, s, top1);
  }
  if (C > kBM) {
    // Experts span several 128-row blocks: several CTAs share each weight
    // tile, and the two-launch kernels, whose static tile order keeps those
    // CTAs in lockstep, measured faster (fewer L2 reads, higher clocks under
    // the power cap).  The fused kernel wins when each weight tile has one user.
    return launch_ffn_two_pass(c, xe, W1, W2, kept_cnt, H, ye, status, s, top1);
  }
  if (!sync_zeroed) {
    cudaError_t e = cudaMemsetAsync(sync, 0, ffn_sync_bytes(c), s);
    if (e != cudaSuccess) return fail(MOE_ERR_CUDA, std::string("cudaMemsetAsync: ") + cudaGetErrorString(e));
  }
  const bool glu = c.expert == MOE_EXPERT_GEGLU;
  const int64_t n1 = glu ? 2 * f : f;  // W1 rows per expert
  CUtensorMap tx, tw1, th, tw2;
  int32_t rc = make_tmap_bf16(&tx, xe, static_cast<uint64_t>(E * C), static_cast<uint64_t>(d), kBM);
  if (rc == MOE_OK) rc = make_tmap_bf16(&tw1, W1, static_cast<uint64_t>(E * n1), static_cast<uint64_t>(d), kBN);
  if (rc == MOE_OK) rc = make_tmap_bf16(&th, H, static_cast<uint64_t>(E * C), static_cast<uint64_t>(f), kBM);
  if (rc == MOE_OK) rc = make_tmap_bf16(&tw2, W2, static_cast<uint64_t>(E * d), static_cast<uint64_t>(f), kBN);
  if (rc != MOE_OK) return rc;
  const int64_t mblk_max = (C + kBM - 1) / kBM;
  const int64_t nb1 = (n1 + kBN - 1) / kBN, nb2 = (d + kBN - 1) / kBN;
  const int64_t g1_per_expert = mblk_max * nb1;
  const int sms = num_sms();
  // lag: GEMM-2 tiles of expert e come after ~2 waves of GEMM-1 tiles of later experts
  const int lag = static_cast<int>(std::min<int64_t>(
      E, std::max<int64_t>(1, (2 * sms + g1_per_expert - 1) / g1_per_expert)));
  FfnParams p{};
  p.E = c.E;
  p.C = c.capacity;
  p.d = c.d_model;
  p.f = c.d_ff;
  p.n1 = static_cast<int>(n1);
  p.glu = glu ? 1 : 0;
  p.lag = lag;
  p.kept_cnt = kept_cnt;
  p.H = static_cast<__nv_bfloat16*>(H);
  p.ye = static_cast<__nv_bfloat16*>(ye);
  p.tile_ctr = static_cast<unsigned int*>(sync);
  p.done1 = static_cast<unsigned int*>(sync) + 1;
  p.status = status;
  p.wait_ns = wait_limit_ns();
  if (top1) {
    p.tok_of_row = top1->tok_of_row;
    p.gate = top1->gate;
    p.y = static_cast<__nv_bfloat16*>(top1->y);
  }
  if (cudaFuncSetAttribute(ffn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           kSmemBytes) != cudaSuccess)
    return check_launch("cudaFuncSetAttribute(ffn_tc_kernel)");
  const int64_t max_tiles = E * mblk_max * (nb1 + nb2);
  const int grid = static_cast<int>(std::min<int64_t>(sms, max_tiles));
  launch_pdl(ffn_tc_kernel, dim3(grid), dim3(kThreads), kSmemBytes, s, tx, tw1, th, tw2, p);
  return check_launch("ffn_tc_kernel");
}

}  // namespace moe
