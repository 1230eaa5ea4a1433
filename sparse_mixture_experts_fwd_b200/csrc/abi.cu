// C ABI entry points: argument validation, workspace layout and the layer
// forward sequence.  Every device-side step is one of the library's kernels.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <mutex>
#include <string>

#include "moe_internal.cuh"

namespace moe {

namespace {
thread_local std::string g_last_error;
std::atomic<uint64_t> g_wait_limit_ns{dev::kDefaultWaitLimitNs};
}

uint64_t wait_limit_ns() { return g_wait_limit_ns.load(std::memory_order_relaxed); }

void set_last_error(const std::string& msg) { g_last_error = msg; }

const char* last_error_cstr() { return g_last_error.c_str(); }

int32_t fail(int32_t code, const std::string& msg) {
  g_last_error = msg;
  return code;
}

int32_t check_launch(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) return MOE_OK;
  return fail(MOE_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

int num_sms() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

namespace {

constexpr int64_t kI32Max = 2147483647;

int32_t check_cfg(const moe_config* c) {
  if (!c) return fail(MOE_ERR_INVALID_ARGUMENT, "config is null");
  if (c->T < 0 || c->T > kI32Max) return fail(MOE_ERR_INVALID_ARGUMENT, "T out of range");
  if (c->E < 1) return fail(MOE_ERR_INVALID_ARGUMENT, "E < 1");
  if (c->E > 256) return fail(MOE_ERR_UNSUPPORTED, "E > 256");
  if (c->k != 1 && c->k != 2) return fail(MOE_ERR_UNSUPPORTED, "k must be 1 or 2");
  if (c->k > c->E) return fail(MOE_ERR_INVALID_ARGUMENT, "k > E");
  if (c->capacity < 0) return fail(MOE_ERR_INVALID_ARGUMENT, "capacity < 0");
  if (c->dtype != MOE_DTYPE_BF16 && c->dtype != MOE_DTYPE_F32)
    return fail(MOE_ERR_INVALID_ARGUMENT, "unknown dtype");
  if (c->mode != MOE_ROUTE_TOPK && c->mode != MOE_ROUTE_RRE)
    return fail(MOE_ERR_INVALID_ARGUMENT, "unknown routing mode");
  if (c->mode == MOE_ROUTE_RRE) {
    if (c->k != 1) return fail(MOE_ERR_INVALID_ARGUMENT, "RRE routes each token to one expert (k=1)");
    if (c->num_groups < 1 || c->E % c->num_groups != 0)
      return fail(MOE_ERR_INVALID_ARGUMENT, "RRE needs num_groups >= 1 dividing E");
  }
  if (c->expert != MOE_EXPERT_RELU && c->expert != MOE_EXPERT_GEGLU)
    return fail(MOE_ERR_INVALID_ARGUMENT, "unknown expert network");
  if (c->reserved != 0) return fail(MOE_ERR_INVALID_ARGUMENT, "reserved field must be 0");
  if (c->expert == MOE_EXPERT_GEGLU && c->dtype != MOE_DTYPE_BF16)
    return fail(MOE_ERR_UNSUPPORTED, "GEGLU experts are bf16 only");
  if (c->d_model < 1 || c->d_ff < 1) return fail(MOE_ERR_INVALID_ARGUMENT, "d_model/d_ff < 1");
  if (c->dtype == MOE_DTYPE_BF16) {
    if (c->d_model % 64 || c->d_ff % 64)
      return fail(MOE_ERR_UNSUPPORTED, "bf16 layers need d_model and d_ff multiples of 64");
  } else {
    if (c->d_model % 4 || c->d_ff % 4)
      return fail(MOE_ERR_UNSUPPORTED, "fp32 layers need d_model and d_ff multiples of 4");
  }
  const int64_t EC = int64_t(c->E) * c->capacity;
  if (EC > kI32Max || int64_t(c->E) * c->d_ff * 2 > kI32Max || int64_t(c->E) * c->d_model > kI32Max)
    return fail(MOE_ERR_UNSUPPORTED, "E*C, E*d_ff or E*d_model exceeds 2^31-1 rows");
  // per-expert arrival counts, slots and the choice index are 32-bit
  if (c->T * c->k > kI32Max) return fail(MOE_ERR_UNSUPPORTED, "T*k exceeds 2^31-1 choices");
  return MOE_OK;
}

int32_t need_ptr(const void* p, const char* name, bool required = true) {
  if (!p) {
    if (!required) return MOE_OK;
    return fail(MOE_ERR_INVALID_ARGUMENT, std::string(name) + " is null");
  }
  if (!aligned16(p)) return fail(MOE_ERR_ALIGNMENT, std::string(name) + " is not 16-byte aligned");
  return MOE_OK;
}

// 4-byte-aligned pointers are enough for the per-token index/gate arrays.
int32_t need_ptr4(const void* p, const char* name) {
  if (!p) return fail(MOE_ERR_INVALID_ARGUMENT, std::string(name) + " is null");
  if (reinterpret_cast<uintptr_t>(p) & 3u)
    return fail(MOE_ERR_ALIGNMENT, std::string(name) + " is not 4-byte aligned");
  return MOE_OK;
}

#define MOE_TRY(expr)              \
  do {                             \
    int32_t rc_ = (expr);          \
    if (rc_ != MOE_OK) return rc_; \
  } while (0)

void layout(const moe_config& c, moe_workspace_map* m) {
  const size_t es = elem_size(c.dtype);
  const size_t T = static_cast<size_t>(c.T), k = static_cast<size_t>(c.k);
  const size_t E = static_cast<size_t>(c.E), C = static_cast<size_t>(c.capacity);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off += align256(bytes);
    return o;
  };
  // bf16 layers fuse the gate into the router, so only fp32 top-k layers keep logits
  m->logits = take(c.mode == MOE_ROUTE_TOPK && c.dtype == MOE_DTYPE_F32 ? T * E * 4 : 0);
  m->expert_idx = take(T * k * 4);
  m->gate = take(T * k * 4);
  m->slot = take(T * k * 4);
  m->kept = take(T * k);
  m->tok_of_row = take(E * C * 4);
  m->arrivals = take(E * 4);
  m->kept_cnt = take(E * 4);
  m->n_dropped = take(4);
  m->scratch = take(assign_scratch_bytes(c));
  m->ffn_sync = take(ffn_sync_bytes(c));
  m->xe = take(E * C * static_cast<size_t>(c.d_model) * es);
  m->H = take(E * C * static_cast<size_t>(c.d_ff) * es);
  m->ye = take(E * C * static_cast<size_t>(c.d_model) * es);
  m->total = off;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

int32_t moe_abi_version(void) { return MOE_ABI_VERSION; }
size_t moe_config_size(void) { return sizeof(moe_config); }
size_t moe_workspace_map_size(void) { return sizeof(moe_workspace_map); }

const char* moe_error_string(int32_t code) {
  switch (code) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARGUMENT: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported configuration";
    case MOE_ERR_ALIGNMENT: return "pointer not aligned";
    case MOE_ERR_WORKSPACE: return "workspace missing or too small";
    case MOE_ERR_CUDA: return "CUDA error";
    default: return "unknown error";
  }
}

const char* moe_last_error(void) { return last_error_cstr(); }

void moe_set_wait_limit_ns(uint64_t ns) {
  g_wait_limit_ns.store(ns == 0 ? dev::kDefaultWaitLimitNs : ns, std::memory_order_relaxed);
}

uint64_t moe_wait_limit_ns(void) { return wait_limit_ns(); }

int32_t moe_bounds_checked(void) { return MOE_CHECK_BOUNDS; }

int32_t moe_capacity(int64_t T, int32_t E, double capacity_factor) {
  if (E < 1 || T < 0 || !(capacity_factor >= 0.0)) return -1;
  const double c = std::floor(static_cast<double>(T) / E * capacity_factor);
  return c > 2147483647.0 ? -1 : static_cast<int32_t>(c);
}

int32_t moe_config_check(const moe_config* cfg) {
  set_last_error("");
  return check_cfg(cfg);
}

size_t moe_assign_workspace_size(const moe_config* cfg) {
  if (check_cfg(cfg) != MOE_OK) return 0;
  return assign_scratch_bytes(*cfg);
}

int32_t moe_workspace_layout(const moe_config* cfg, moe_workspace_map* out) {
  set_last_error("");
  MOE_TRY(check_cfg(cfg));
  if (!out) return fail(MOE_ERR_INVALID_ARGUMENT, "out is null");
  layout(*cfg, out);
  return MOE_OK;
}

size_t moe_workspace_size(const moe_config* cfg) {
  if (check_cfg(cfg) != MOE_OK) return 0;
  moe_workspace_map m;
  layout(*cfg, &m);
  return m.total;
}

int32_t moe_router(const moe_config* cfg, const void* x, const void* Wr, const float* bias,
                   float* logits, int32_t* status, moe_stream_t stream) {
  CallRange range_("moe_router");
  set_last_error("");
  MOE_TRY(check_cfg(cfg));
  if (cfg->T == 0) return MOE_OK;
  MOE_TRY(need_ptr(x, "x"));
  MOE_TRY(need_ptr(Wr, "Wr"));
  MOE_TRY(need_ptr(bias, "bias", false));
  MOE_TRY(need_ptr(logits, "logits"));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cfg->dtype == MOE_DTYPE_BF16) return launch_router_tc(*cfg, x, Wr, bias, logits, status, s);
  return launch_router_f32(*cfg, x, Wr, bias, logits, s);
}

int32_t moe_topk_assign(const moe_config* cfg, const float* logits, const int32_t* domain_id,
                        int32_t* expert_idx, float* gate, int32_t* slot, uint8_t* kept,
                        int32_t* tok_of_row, int32_t* arrivals, int32_t* kept_cnt,
                        int32_t* n_dropped, void* workspace, size_t workspace_bytes,
                        int32_t* status, moe_stream_t stream) {
  CallRange range_("moe_topk_assign");
  set_last_error("");
  MOE_TRY(check_cfg(cfg));
  const bool any_tokens = cfg->T > 0;
  if (any_tokens) {
    if (cfg->mode == MOE_ROUTE_TOPK) MOE_TRY(need_ptr4(logits, "logits"));
    else MOE_TRY(need_ptr4(domain_id, "domain_id"));
    MOE_TRY(need_ptr4(expert_idx, "expert_idx"));
    MOE_TRY(need_ptr4(gate, "gate"));
    MOE_TRY(need_ptr4(slot, "slot"));
    if (!kept) return fail(MOE_ERR_INVALID_ARGUMENT, "kept is null");
  }
  if (int64_t(cfg->E) * cfg->capacity > 0) MOE_TRY(need_ptr4(tok_of_row, "tok_of_row"));
  MOE_TRY(need_ptr4(arrivals, "arrivals"));
  MOE_TRY(need_ptr4(kept_cnt, "kept_cnt"));
  MOE_TRY(need_ptr4(n_dropped, "n_dropped"));
  const size_t need = assign_scratch_bytes(*cfg);
  if (need > 0 && (!workspace || workspace_bytes < need))
    return fail(MOE_ERR_WORKSPACE, "moe_topk_assign: workspace needs " + std::to_string(need) + " bytes");
  if (workspace) MOE_TRY(need_ptr(workspace, "workspace"));
  return launch_route_assign(*cfg, logits, domain_id, expert_idx, gate, slot, kept, tok_of_row,
                             arrivals, kept_cnt, n_dropped, workspace, status,
                             reinterpret_cast<cudaStream_t>(stream));
}

int32_t moe_dispatch(const moe_config* cfg, const void* x, const int32_t* expert_idx,
                     const int32_t* slot, const uint8_t* kept, void* xe, int32_t* status,
                     moe_stream_t stream) {
  CallRange range_("moe_dispatch");
  set_last_error("");
  MOE_TRY(check_cfg(cfg));
  if (cfg->T == 0 || cfg->capacity == 0) return MOE_OK;
  MOE_TRY(need_ptr(x, "x"));
  MOE_TRY(need_ptr4(expert_idx, "expert_idx"));
  MOE_TRY(need_ptr4(slot, "slot"));
  if (!kept) return fail(MOE_ERR_INVALID_ARGUMENT, "kept is null");
  MOE_TRY(need_ptr(xe, "xe"));
  return launch_dispatch(*cfg, x, expert_idx, slot, kept, xe, status,
                         reinterpret_cast<cudaStream_t>(stream));
}

size_t moe_ffn_workspace_size(const moe_config* cfg) {
  if (check_cfg(cfg) != MOE_OK) return 0;
  return ffn_sync_bytes(*cfg);
}

int32_t moe_expert_ffn(const moe_config* cfg, const void* xe, const void* W1, const void* W2,
                       const int32_t* kept_cnt, void* H, void* ye, void* workspace,
                       size_t workspace_bytes, int32_t* status, moe_stream_t stream) {
  return moe_expert_ffn_ex(cfg, xe, W1, W2, kept_cnt, H, ye, workspace, workspace_bytes, 0u,
                           status, stream);
}

int32_t moe_expert_ffn_ex(const moe_config* cfg, const void* xe, const void* W1, const void* W2,
                          const int32_t* kept_cnt, void* H, void* ye, void* workspace,
                          size_t workspace_bytes, uint32_t flags, int32_t* status,
                          moe_stream_t stream) {
  CallRange range_("moe_expert_ffn_ex");
  set_last_error("");
  if (flags & ~static_cast<uint32_t>(MOE_FFN_WORKSPACE_ZEROED))
    return fail(MOE_ERR_INVALID_ARGUMENT, "moe_expert_ffn_ex: unknown flag bits");
  MOE_TRY(check_cfg(cfg));
  if (cfg->capacity == 0) return MOE_OK;
  MOE_TRY(need_ptr(xe, "xe"));
  MOE_TRY(need_ptr(W1, "W1"));
  MOE_TRY(need_ptr(W2, "W2"));
  MOE_TRY(need_ptr4(kept_cnt, "kept_cnt"));
  MOE_TRY(need_ptr(H, "H"));
  MOE_TRY(need_ptr(ye, "ye"));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cfg->dtype == MOE_DTYPE_BF16) {
    const size_t need = ffn_sync_bytes(*cfg);
    if (!workspace || workspace_bytes < need)
      return fail(MOE_ERR_WORKSPACE, "moe_expert_ffn: workspace needs " + std::to_string(need) + " bytes");
    MOE_TRY(need_ptr(workspace, "workspace"));
    return launch_ffn_tc(*cfg, xe, W1, W2, kept_cnt, H, ye, workspace,
                         (flags & MOE_FFN_WORKSPACE_ZEROED) != 0, status, s);
  }
  return launch_ffn_f32(*cfg, xe, W1, W2, kept_cnt, H, ye, s);
}

int32_t moe_combine(const moe_config* cfg, const void* ye, const int32_t* expert_idx,
                    const float* gate, const int32_t* slot, const uint8_t* kept, void* y,
                    int32_t* status, moe_stream_t stream) {
  CallRange range_("moe_combine");
  set_last_error("");
  MOE_TRY(check_cfg(cfg));
  if (cfg->T == 0) return MOE_OK;
  if (cfg->capacity > 0) MOE_TRY(need_ptr(ye, "ye"));
  MOE_TRY(need_ptr4(expert_idx, "expert_idx"));
  MOE_TRY(need_ptr4(gate, "gate"));
  MOE_TRY(need_ptr4(slot, "slot"));
  if (!kept) return fail(MOE_ERR_INVALID_ARGUMENT, "kept is null");
  MOE_TRY(need_ptr(y, "y"));
  return launch_combine(*cfg, ye, expert_idx, gate, slot, kept, y, status,
                        reinterpret_cast<cudaStream_t>(stream));
}

size_t moe_aux_workspace_size(const moe_config* cfg) {
  if (check_cfg(cfg) != MOE_OK) return 0;
  return aux_workspace_bytes(*cfg);
}

int32_t moe_aux_loss(const moe_config* cfg, const float* logits, double alpha, double* out,
                     double* f, double* P, void* workspace, size_t workspace_bytes,
                     moe_stream_t stream) {
  CallRange range_("moe_aux_loss");
  set_last_error("");
  MOE_TRY(check_cfg(cfg));
  if (cfg->mode != MOE_ROUTE_TOPK)
    return fail(MOE_ERR_UNSUPPORTED, "moe_aux_loss: RRE routing has no learned gate");
  if (cfg->T > 0) MOE_TRY(need_ptr4(logits, "logits"));
  auto need8 = [](const void* q, const char* name, bool required) -> int32_t {
    if (!q) return required ? fail(MOE_ERR_INVALID_ARGUMENT, std::string(name) + " is null") : MOE_OK;
    if (reinterpret_cast<uintptr_t>(q) & 7u)
      return fail(MOE_ERR_ALIGNMENT, std::string(name) + " is not 8-byte aligned");
    return MOE_OK;
  };
  MOE_TRY(need8(out, "out", true));
  MOE_TRY(need8(f, "f", false));
  MOE_TRY(need8(P, "P", false));
  const size_t need = aux_workspace_bytes(*cfg);
  if (!workspace || workspace_bytes < need)
    return fail(MOE_ERR_WORKSPACE, "moe_aux_loss: workspace needs " + std::to_string(need) + " bytes");
  MOE_TRY(need_ptr(workspace, "workspace"));
  return launch_aux_loss(*cfg, logits, alpha, out, f, P, workspace,
                         reinterpret_cast<cudaStream_t>(stream));
}

int32_t moe_layer_forward(const moe_config* cfg, const void* x, const void* Wr, const float* bias,
                          const int32_t* domain_id, const void* W1, const void* W2, void* y,
                          void* workspace, size_t workspace_bytes, int32_t* status,
                          void* const* stage_events, moe_stream_t stream) {
  CallRange range_("moe_layer_forward");
  set_last_error("");
  MOE_TRY(check_cfg(cfg));
  const moe_config& c = *cfg;
  moe_workspace_map m;
  layout(c, &m);
  if (!workspace || workspace_bytes < m.total)
    return fail(MOE_ERR_WORKSPACE, "moe_layer_forward: workspace needs " + std::to_string(m.total) + " bytes");
  MOE_TRY(need_ptr(workspace, "workspace"));
  if (c.T > 0) {
    MOE_TRY(need_ptr(x, "x"));
    MOE_TRY(need_ptr(y, "y"));
    if (c.mode == MOE_ROUTE_TOPK) {
      MOE_TRY(need_ptr(Wr, "Wr"));
      MOE_TRY(need_ptr(bias, "bias", false));
    } else {
      MOE_TRY(need_ptr4(domain_id, "domain_id"));
    }
  }
  if (c.capacity > 0) {
    MOE_TRY(need_ptr(W1, "W1"));
    MOE_TRY(need_ptr(W2, "W2"));
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  float* logits = reinterpret_cast<float*>(ws + m.logits);
  int32_t* expert_idx = reinterpret_cast<int32_t*>(ws + m.expert_idx);
  float* gate = reinterpret_cast<float*>(ws + m.gate);
  int32_t* slot = reinterpret_cast<int32_t*>(ws + m.slot);
  uint8_t* kept = reinterpret_cast<uint8_t*>(ws + m.kept);
  int32_t* tok_of_row = reinterpret_cast<int32_t*>(ws + m.tok_of_row);
  int32_t* arrivals = reinterpret_cast<int32_t*>(ws + m.arrivals);
  int32_t* kept_cnt = reinterpret_cast<int32_t*>(ws + m.kept_cnt);
  int32_t* n_dropped = reinterpret_cast<int32_t*>(ws + m.n_dropped);
  void* scratch = ws + m.scratch;
  void* xe = ws + m.xe;
  void* H = ws + m.H;
  void* ye = ws + m.ye;

  auto mark = [&](int i) -> int32_t {
    if (!stage_events || !stage_events[i]) return MOE_OK;
    cudaError_t e = cudaEventRecord(static_cast<cudaEvent_t>(stage_events[i]), s);
    return e == cudaSuccess ? MOE_OK
                            : fail(MOE_ERR_CUDA, std::string("cudaEventRecord: ") + cudaGetErrorString(e));
  };
  // the fused expert FFN's counters are cleared by the dispatch kernel
  unsigned int* ffn_sync = reinterpret_cast<unsigned int*>(ws + m.ffn_sync);
  const bool dispatch_zeroes = c.T > 0 && c.capacity > 0 && c.dtype == MOE_DTYPE_BF16;
  const int n_sync_words = static_cast<int>(ffn_sync_bytes(c) / sizeof(unsigned int));

  MOE_TRY(mark(0));
  const bool fused_router = c.mode == MOE_ROUTE_TOPK && c.dtype == MOE_DTYPE_BF16 && c.T > 0;
  if (fused_router) {
    // router GEMM with the gate and top-k in its epilogue (no logits round trip)
    MOE_TRY(launch_router_topk_tc(c, x, Wr, bias, expert_idx, gate, status, s));
  } else if (c.mode == MOE_ROUTE_TOPK && c.T > 0) {
    MOE_TRY(launch_router_f32(c, x, Wr, bias, logits, s));
  }
  MOE_TRY(mark(1));
  if (fused_router)
    MOE_TRY(launch_assign(c, expert_idx, slot, kept, tok_of_row, arrivals, kept_cnt, n_dropped,
                          scratch, status, s));
  else
    MOE_TRY(launch_route_assign(c, logits, domain_id, expert_idx, gate, slot, kept, tok_of_row,
                                arrivals, kept_cnt, n_dropped, scratch, status, s));
  MOE_TRY(mark(2));
  // Top-1 bf16 layers combine inside the expert FFN: its second GEMM writes
  // gate * row straight into y (token order) and the dispatch kernel zeroes the
  // rows of dropped tokens, so ye is not materialised and no combine runs.
  const bool fused_combine = c.k == 1 && c.dtype == MOE_DTYPE_BF16 && c.T > 0;
  const Top1Out top1{tok_of_row, gate, y};
  MOE_TRY(launch_dispatch(c, x, expert_idx, slot, kept, xe, status, s,
                          dispatch_zeroes ? ffn_sync : nullptr, dispatch_zeroes ? n_sync_words : 0,
                          fused_combine ? y : nullptr));
  MOE_TRY(mark(3));
  if (c.dtype == MOE_DTYPE_BF16)
    MOE_TRY(launch_ffn_tc(c, xe, W1, W2, kept_cnt, H, ye, ffn_sync, dispatch_zeroes, status, s,
                          fused_combine ? &top1 : nullptr));
  else MOE_TRY(launch_ffn_f32(c, xe, W1, W2, kept_cnt, H, ye, s));
  MOE_TRY(mark(4));
  if (!fused_combine) MOE_TRY(launch_combine(c, ye, expert_idx, gate, slot, kept, y, status, s));
  return mark(5);
}

namespace {

int32_t check_ep(const moe_config* cfg, int32_t rank, int32_t world) {
  MOE_TRY(check_cfg(cfg));
  if (world < 1 || world > kMaxEpRanks)
    return fail(MOE_ERR_INVALID_ARGUMENT, "world must be 1.." + std::to_string(kMaxEpRanks));
  if (rank < 0 || rank >= world) return fail(MOE_ERR_INVALID_ARGUMENT, "rank outside 0..world-1");
  if (cfg->E % world != 0) return fail(MOE_ERR_INVALID_ARGUMENT, "world does not divide E");
  if (int64_t(world) * cfg->capacity > kI32Max)
    return fail(MOE_ERR_UNSUPPORTED, "world * capacity exceeds 2^31-1 rows");
  return MOE_OK;
}

int32_t check_peers(const void* const* peers, int32_t world, const char* name) {
  if (!peers) return fail(MOE_ERR_INVALID_ARGUMENT, std::string(name) + " is null");
  for (int q = 0; q < world; ++q)
    MOE_TRY(need_ptr(peers[q], (std::string(name) + "[" + std::to_string(q) + "]").c_str()));
  return MOE_OK;
}

}  // namespace

int32_t moe_ep_ffn_config(const moe_config* cfg, int32_t world, moe_config* out) {
  set_last_error("");
  MOE_TRY(check_ep(cfg, 0, world));
  if (!out) return fail(MOE_ERR_INVALID_ARGUMENT, "out is null");
  moe_config c = *cfg;
  c.E = cfg->E / world;
  c.capacity = world * cfg->capacity;
  c.k = 1;
  c.mode = MOE_ROUTE_TOPK;
  c.num_groups = 1;
  MOE_TRY(check_cfg(&c));
  *out = c;
  return MOE_OK;
}

int32_t moe_ep_dispatch(const moe_config* cfg, int32_t rank, int32_t world, const void* x,
                        const int32_t* expert_idx, const int32_t* slot, const uint8_t* kept,
                        const int32_t* cnt_all, void* const* xe_peers, int32_t* local_cnt,
                        int32_t* status, moe_stream_t stream) {
  CallRange range_("moe_ep_dispatch");
  set_last_error("");
  MOE_TRY(check_ep(cfg, rank, world));
  MOE_TRY(need_ptr4(cnt_all, "cnt_all"));
  if (local_cnt) MOE_TRY(need_ptr4(local_cnt, "local_cnt"));
  if (cfg->T > 0 && cfg->capacity > 0) {
    MOE_TRY(need_ptr(x, "x"));
    MOE_TRY(need_ptr4(expert_idx, "expert_idx"));
    MOE_TRY(need_ptr4(slot, "slot"));
    if (!kept) return fail(MOE_ERR_INVALID_ARGUMENT, "kept is null");
    MOE_TRY(check_peers(xe_peers, world, "xe_peers"));
  } else if (!local_cnt) {
    return MOE_OK;  // nothing to send and nothing to count
  }
  moe_config c = *cfg;
  if (c.capacity == 0) c.T = 0;  // no choice is kept
  return launch_ep_dispatch(c, rank, world, x, expert_idx, slot, kept, cnt_all, xe_peers,
                            local_cnt, status, reinterpret_cast<cudaStream_t>(stream));
}

int32_t moe_ep_combine(const moe_config* cfg, int32_t rank, int32_t world,
                       const void* const* ye_peers, const int32_t* expert_idx, const float* gate,
                       const int32_t* slot, const uint8_t* kept, const int32_t* cnt_all, void* y,
                       int32_t* status, moe_stream_t stream) {
  CallRange range_("moe_ep_combine");
  set_last_error("");
  MOE_TRY(check_ep(cfg, rank, world));
  if (cfg->T == 0) return MOE_OK;
  MOE_TRY(need_ptr4(expert_idx, "expert_idx"));
  MOE_TRY(need_ptr4(gate, "gate"));
  MOE_TRY(need_ptr4(slot, "slot"));
  if (!kept) return fail(MOE_ERR_INVALID_ARGUMENT, "kept is null");
  MOE_TRY(need_ptr4(cnt_all, "cnt_all"));
  MOE_TRY(need_ptr(y, "y"));
  if (cfg->capacity > 0) MOE_TRY(check_peers(ye_peers, world, "ye_peers"));
  return launch_ep_combine(*cfg, rank, world, ye_peers, expert_idx, gate, slot, kept, cnt_all, y,
                           status, reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"
