// C ABI of libmoe (declared in include/moe.h): host-side argument validation, the
// workspace layout, and the launch sequence of each step and of the fused forward.
#include <cudaTypedefs.h>
#include <string.h>

#include <mutex>

#include "internal.h"
#include "moe.h"

namespace moe {
namespace {

thread_local int32_t g_last_launches = 0;

constexpr size_t kAlign = 256;
size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int esize(const moe_config* c) { return c->dtype == MOE_BF16 ? 2 : 4; }


// Structural validity of the config (MOE_ERR_INVALID_ARG) and supported shapes
// (MOE_ERR_UNSUPPORTED).
moe_status check_config(const moe_config* c) {
  if (c == nullptr) return MOE_ERR_INVALID_ARG;
  if (c->T < 0 || c->d_model <= 0 || c->d_ff <= 0 || c->E <= 0 || c->k <= 0 || c->k > c->E)
    return MOE_ERR_INVALID_ARG;
  if (c->gating != MOE_GATE_SOFTMAX_TOPK && c->gating != MOE_GATE_NOISY_TOPK &&
      c->gating != MOE_GATE_HIERARCHICAL)
    return MOE_ERR_INVALID_ARG;
  if (c->gating == MOE_GATE_HIERARCHICAL) {
    if (c->groups <= 0 || c->E % c->groups != 0 || c->k_primary <= 0 ||
        c->k_primary > c->groups || c->k % c->k_primary != 0 ||
        c->k / c->k_primary > c->E / c->groups)
      return MOE_ERR_INVALID_ARG;
    if (c->k_primary > 4 || c->k / c->k_primary > 4) return MOE_ERR_UNSUPPORTED;
    if (c->groups + c->E > (c->dtype == MOE_BF16 ? 256 : 1024)) return MOE_ERR_UNSUPPORTED;
  }
  if (c->act != MOE_ACT_RELU && c->act != MOE_ACT_GELU) return MOE_ERR_INVALID_ARG;
  if (c->dtype != MOE_F32 && c->dtype != MOE_BF16) return MOE_ERR_INVALID_ARG;
  if (!(c->capacity_factor == c->capacity_factor)) return MOE_ERR_INVALID_ARG;  // NaN
  if (c->hidden_f16 != 0 && c->hidden_f16 != 1) return MOE_ERR_INVALID_ARG;
  if (c->y_bf16 != 0 && c->y_bf16 != 1) return MOE_ERR_INVALID_ARG;
  if (c->y_bf16 != 0 && c->dtype != MOE_BF16) return MOE_ERR_INVALID_ARG;
  if (c->k > 8) return MOE_ERR_UNSUPPORTED;
  if (c->T * static_cast<int64_t>(c->k) >= (int64_t{1} << 31)) return MOE_ERR_UNSUPPORTED;
  if (c->T * static_cast<int64_t>(c->E) >= (int64_t{1} << 31)) return MOE_ERR_UNSUPPORTED;
  if (c->d_model % 8 != 0) return MOE_ERR_UNSUPPORTED;
  if (c->dtype == MOE_BF16) {
    if (c->d_model % 64 != 0 || c->d_ff % 64 != 0 || c->E > 256) return MOE_ERR_UNSUPPORTED;
  } else {
    if (c->d_ff % 4 != 0 || c->E > 1024) return MOE_ERR_UNSUPPORTED;
  }
  return MOE_OK;
}

struct Layout {
  size_t err, blk, partials, logits, nz, lw, sw, hw, kw, steps;  // step workspace
  size_t offsets, slot_pos, perm_src, x_perm, h, y_perm, forward;  // + forward intermediates
};

Layout layout(const moe_config* c) {
  Layout L;
  const int64_t n = c->T * c->k;
  size_t o = 0;
  L.err = o;
  o = align_up(o + 16);
  L.blk = o;
  o = align_up(o + static_cast<size_t>(permute_count_ints(n, c->E)) * 4);
  L.partials = o;
  o = align_up(o + static_cast<size_t>(route_blocks(c->T)) * 2 * c->E * 4);
  L.logits = o;
  L.nz = o;
  if (c->dtype == MOE_F32) {
    const size_t cols = c->E + (c->gating == MOE_GATE_HIERARCHICAL ? c->groups : 0);
    o = align_up(o + static_cast<size_t>(c->T) * cols * 4);
    L.nz = o;
    if (c->gating == MOE_GATE_NOISY_TOPK) o = align_up(o + static_cast<size_t>(c->T) * c->E * 4);
  }
  L.lw = L.sw = L.hw = L.kw = o;
  if (c->dtype == MOE_BF16 && c->gating == MOE_GATE_NOISY_TOPK) {
    // the per-token values the Importance/Load sums are formed from
    o = align_up(o + static_cast<size_t>(c->T) * c->E * 4);
    L.sw = o;
    o = align_up(o + static_cast<size_t>(c->T) * c->E * 4);
    L.hw = o;
    o = align_up(o + static_cast<size_t>(c->T) * c->E * 4);
    L.kw = o;
    o = align_up(o + static_cast<size_t>(c->T) * 2 * 4);
  }
  L.steps = o;
  L.offsets = o;
  o = align_up(o + static_cast<size_t>(c->E + 1) * 4);
  L.slot_pos = o;
  o = align_up(o + static_cast<size_t>(n) * 4);
  L.perm_src = o;
  o = align_up(o + static_cast<size_t>(n) * 4);
  L.x_perm = o;
  o = align_up(o + static_cast<size_t>(n) * c->d_model * esize(c));
  L.h = o;
  o = align_up(o + static_cast<size_t>(n) * c->d_ff * esize(c));
  L.y_perm = o;
  o = align_up(o + static_cast<size_t>(n) * c->d_model * 4);
  L.forward = o;
  return L;
}

// The forward state moe_forward_train keeps for moe_backward.
// The router's scores are kept expert-major ([E, T]) as the gate wrote them: clean
// logits (+ bias) in lg, and for noisy gating Softplus(x.W_noise) in sw, the noisy scores
// H in hw and the k-th / (k+1)-th H of each token [2, T] in kw.
struct TrainLayout {
  size_t offsets, slot_pos, perm_src, x_perm, u, h, y_perm, lg, sw, hw, kw, total;
};

TrainLayout train_layout(const moe_config* c) {
  TrainLayout L;
  const int64_t n = c->T * c->k;
  size_t o = 0;
  L.offsets = o;
  o = align_up(o + static_cast<size_t>(c->E + 1) * 4);
  L.slot_pos = o;
  o = align_up(o + static_cast<size_t>(n) * 4);
  L.perm_src = o;
  o = align_up(o + static_cast<size_t>(n) * 4);
  L.x_perm = o;
  o = align_up(o + static_cast<size_t>(n) * c->d_model * 2);
  L.u = o;
  o = align_up(o + static_cast<size_t>(n) * c->d_ff * 2);
  L.h = o;
  o = align_up(o + static_cast<size_t>(n) * c->d_ff * 2);
  L.y_perm = o;
  o = align_up(o + static_cast<size_t>(n) * c->d_model * 4);
  const size_t TE = static_cast<size_t>(c->T) * c->E;
  L.lg = o;
  o = align_up(o + TE * 4);
  L.sw = L.hw = L.kw = o;
  if (c->gating == MOE_GATE_NOISY_TOPK) {
    o = align_up(o + TE * 4);
    L.hw = o;
    o = align_up(o + TE * 4);
    L.kw = o;
    o = align_up(o + static_cast<size_t>(c->T) * 2 * 4);
  }
  L.total = o;
  return L;
}

// moe_backward's workspace: the step workspace (error word first), then its buffers.
struct BackwardLayout {
  size_t poff, d_o, du, dx_perm, dl, dimp, dload, part, total;  // dz follows dl
  int64_t part_cap;
};

BackwardLayout backward_layout(const moe_config* c, size_t steps) {
  BackwardLayout L;
  const int64_t n = c->T * c->k;
  const int64_t prows = backward_padded_rows(n, c->E);
  const size_t TE = static_cast<size_t>(c->T) * c->E;
  size_t o = steps;
  L.poff = o;
  o = align_up(o + static_cast<size_t>(c->E + 1) * 4);
  L.d_o = o;
  o = align_up(o + static_cast<size_t>(prows) * c->d_model * 2);
  L.du = o;
  o = align_up(o + static_cast<size_t>(prows) * c->d_ff * 2);
  L.dx_perm = o;
  o = align_up(o + static_cast<size_t>(n) * c->d_model * 4);
  L.dl = o;  // [E, T], for noisy gating followed by dz [E, T]
  o = align_up(o + TE * 4 * (c->gating == MOE_GATE_NOISY_TOPK ? 2 : 1));
  L.dimp = o;
  o = align_up(o + static_cast<size_t>(c->E) * 4);
  L.dload = o;
  o = align_up(o + static_cast<size_t>(c->E) * 4);
  L.part = o;
  const int64_t a = 64LL * c->E * c->d_model, b = 4LL * c->T * c->E;
  L.part_cap = a > b ? a : b;
  o = align_up(o + static_cast<size_t>(L.part_cap) * 4);
  L.total = o;
  return L;
}

// Configurations the training forward and the backward support: bf16 layers with the
// softmax or noisy gate.
moe_status check_train_config(const moe_config* c) {
  moe_status st = check_config(c);
  if (st != MOE_OK) return st;
  if (c->dtype != MOE_BF16 || c->gating == MOE_GATE_HIERARCHICAL) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

int64_t capacity_of(const moe_config* c) {
  const float cf = c->capacity_factor;
  if (!(cf > 0.0f)) return -1;
  // exact ceil(cf * T * k / E) with cf = m * 2^ex, m a 24-bit integer
  int ex = 0;
  const double fr = frexp(static_cast<double>(cf), &ex);  // cf = fr * 2^ex, fr in [0.5, 1)
  const uint64_t m = static_cast<uint64_t>(ldexp(fr, 24));  // exact for a float
  ex -= 24;                                                 // cf = m * 2^ex
  unsigned __int128 num = static_cast<unsigned __int128>(m) * static_cast<uint64_t>(c->T) *
                          static_cast<uint64_t>(c->k);
  unsigned __int128 den = static_cast<unsigned __int128>(c->E);
  if (ex >= 0) {
    if (ex > 60) return INT64_MAX;
    num <<= ex;
  } else {
    if (-ex > 60) den <<= 60; else den <<= -ex;
  }
  const unsigned __int128 q = (num + den - 1) / den;
  return q > static_cast<unsigned __int128>(INT64_MAX) ? INT64_MAX : static_cast<int64_t>(q);
}

struct Ctx {
  LaunchCtx lc;
  int launches = 0;
  bool ok = false;
  Ctx(void* ws, moe_stream_t stream) {
    lc.stream = reinterpret_cast<cudaStream_t>(stream);
    lc.err = reinterpret_cast<int*>(ws);
    lc.launches = &launches;
    int dev = 0;
    ok = cudaGetDevice(&dev) == cudaSuccess &&
         cudaDeviceGetAttribute(&lc.num_sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess;
  }
  moe_status finish(cudaError_t e) {
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    g_last_launches = launches;
    return MOE_OK;
  }
};

// keep (training only, or null): the train state's base; the gate then writes the
// router's scores into its lg / sw / hw / kw buffers for the backward.
moe_status do_route(const moe_config* cfg, const Layout& L, const void* x, const void* w_gate,
                    const void* w_noise, const float* noise, const float* logit_bias,
                    int32_t* topk_idx, float* topk_gate, float* importance, float* load,
                    uint8_t* near_tie, void* ws, Ctx& ctx, uint8_t* keep = nullptr) {
  uint8_t* w = static_cast<uint8_t*>(ws);
  RouteProblem p;
  p.T = cfg->T;
  p.d = cfg->d_model;
  p.E = cfg->E;
  p.k = cfg->k;
  p.noisy = cfg->gating == MOE_GATE_NOISY_TOPK;
  p.renorm = cfg->renorm != 0;
  p.hier = cfg->gating == MOE_GATE_HIERARCHICAL;
  p.groups = p.hier ? cfg->groups : 0;
  p.k_primary = p.hier ? cfg->k_primary : 0;
  p.bias = p.hier ? nullptr : logit_bias;
  p.x = x;
  p.w_gate = w_gate;
  p.w_noise = w_noise;
  p.noise = noise;
  p.topk_idx = topk_idx;
  p.topk_gate = topk_gate;
  p.near_tie = near_tie;
  p.importance = importance;
  p.load = load;
  p.partials = reinterpret_cast<float*>(w + L.partials);
  p.logits_ws = reinterpret_cast<float*>(w + L.logits);
  p.nz_ws = reinterpret_cast<float*>(w + L.nz);
  if (keep != nullptr) {
    const TrainLayout S = train_layout(cfg);
    p.lw = reinterpret_cast<float*>(keep + S.lg);
    p.sw = reinterpret_cast<float*>(keep + S.sw);
    p.hw = reinterpret_cast<float*>(keep + S.hw);
    p.kw = reinterpret_cast<float*>(keep + S.kw);
    p.store_scores = true;
  } else if (cfg->dtype == MOE_BF16 && cfg->gating == MOE_GATE_NOISY_TOPK) {
    p.lw = reinterpret_cast<float*>(w + L.lw);
    p.sw = reinterpret_cast<float*>(w + L.sw);
    p.hw = reinterpret_cast<float*>(w + L.hw);
    p.kw = reinterpret_cast<float*>(w + L.kw);
  }
  cudaError_t e = cfg->dtype == MOE_BF16 ? launch_route_bf16(p, ctx.lc) : launch_route_f32(p, ctx.lc);
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status check_route_args(const moe_config* cfg, const void* x, const void* w_gate,
                            const void* w_noise, const float* noise, const int32_t* topk_idx,
                            const float* topk_gate, const float* importance, const float* load,
                            const void* ws) {
  if (!x || !w_gate || !topk_idx || !topk_gate || !ws) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w_gate) || !aligned16(ws)) return MOE_ERR_INVALID_ARG;
  const bool noisy = cfg->gating == MOE_GATE_NOISY_TOPK;
  if (noisy && (!w_noise || !noise || !aligned16(w_noise))) return MOE_ERR_INVALID_ARG;
  if (load && !(noisy && cfg->k < cfg->E)) return MOE_ERR_INVALID_ARG;
  if (cfg->gating == MOE_GATE_HIERARCHICAL && importance) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

moe_status do_permute(const moe_config* cfg, const Layout& L, const int32_t* topk_idx,
                      const void* x, int32_t* counts, int32_t* offsets, int32_t* perm_src,
                      int32_t* slot_pos, void* x_perm, void* ws, Ctx& ctx) {
  PermuteProblem p;
  p.n = cfg->T * cfg->k;
  p.k = cfg->k;
  p.E = cfg->E;
  p.d = cfg->d_model;
  p.esize = esize(cfg);
  p.C = capacity_of(cfg);
  p.topk_idx = topk_idx;
  p.x = x;
  p.counts = counts;
  p.offsets = offsets;
  p.perm_src = perm_src;
  p.slot_pos = slot_pos;
  p.x_perm = x_perm;
  p.blk = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(ws) + L.blk);
  p.ticket = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(ws) + L.err + 8);
  p.sync = p.ticket;  // words 2 and 3 of the error block, zero between calls
  return launch_permute(p, ctx.lc) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// x_perm: the permuted rows; or, with gather_src, x is the token rows and permuted row s
// reads x[gather_src[s] / k].
moe_status do_ffn(const moe_config* cfg, const void* x_perm, const int32_t* offsets, const void* w1,
                  const void* w2, void* h, void* y_perm, Ctx& ctx, const void* x = nullptr,
                  const int32_t* gather_src = nullptr, void* u = nullptr) {
  FfnProblem p;
  p.u = u;
  p.x = x;
  p.gather_src = gather_src;
  p.x_rows = cfg->T;
  p.k = cfg->k;
  p.rows_cap = cfg->T * cfg->k;
  p.d = cfg->d_model;
  p.f = cfg->d_ff;
  p.E = cfg->E;
  p.act = cfg->act == MOE_ACT_GELU ? 2 : 1;
  p.hidden_f16 = cfg->dtype == MOE_BF16 && cfg->hidden_f16;
  p.x_perm = x_perm;
  p.offsets = offsets;
  p.w1 = w1;
  p.w2 = w2;
  p.h = h;
  p.y_perm = y_perm;
  cudaError_t e = cfg->dtype == MOE_BF16 ? launch_ffn_bf16(p, ctx.lc) : launch_ffn_f32(p, ctx.lc);
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status do_combine(const moe_config* cfg, const void* y_perm, const int32_t* slot_pos,
                      const float* gate, void* y, Ctx& ctx) {
  CombineProblem p;
  p.T = cfg->T;
  p.k = cfg->k;
  p.d = cfg->d_model;
  p.y_perm = y_perm;
  p.slot_pos = slot_pos;
  p.gate = gate;
  p.y = y;
  p.y_bf16 = cfg->y_bf16;
  return launch_combine(p, ctx.lc) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status do_ffn_combine(const moe_config* cfg, const void* x_perm, const int32_t* offsets,
                          const int32_t* perm_src, const int32_t* slot_pos, const float* gate,
                          const void* w1, const void* w2, void* h, void* y, Ctx& ctx,
                          const void* x = nullptr, bool gather = false) {
  FfnProblem p;
  p.x = x;
  p.gather_src = gather ? perm_src : nullptr;
  p.x_rows = cfg->T;
  p.k = cfg->k;
  p.rows_cap = cfg->T * cfg->k;
  p.d = cfg->d_model;
  p.f = cfg->d_ff;
  p.E = cfg->E;
  p.act = cfg->act == MOE_ACT_GELU ? 2 : 1;
  p.hidden_f16 = cfg->hidden_f16;
  p.x_perm = x_perm;
  p.offsets = offsets;
  p.w1 = w1;
  p.w2 = w2;
  p.h = h;
  p.y_perm = nullptr;
  p.y_bf16 = cfg->y_bf16;
  cudaError_t e = launch_ffn_combine_bf16(p, perm_src, slot_pos, gate, y, ctx.lc);
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// FFN and combine as one step: bf16 with k = 1 (the combine is a scaled store), or k = 2
// with an fp32 y (two in-memory adds per row, which commute)
bool fused_combine(const moe_config* cfg) {
  return cfg->dtype == MOE_BF16 && (cfg->k == 1 || (cfg->k == 2 && !cfg->y_bf16));
}

// T == 0: nothing to route; zero the per-expert outputs that are defined anyway.
moe_status empty_batch(const moe_config* cfg, int32_t* counts, int32_t* offsets, float* importance,
                       float* load, moe_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const size_t E = static_cast<size_t>(cfg->E);
  if (counts && cudaMemsetAsync(counts, 0, E * 4, s) != cudaSuccess) return MOE_ERR_CUDA;
  if (offsets && cudaMemsetAsync(offsets, 0, (E + 1) * 4, s) != cudaSuccess) return MOE_ERR_CUDA;
  if (importance && cudaMemsetAsync(importance, 0, E * 4, s) != cudaSuccess) return MOE_ERR_CUDA;
  if (load && cudaMemsetAsync(load, 0, E * 4, s) != cudaSuccess) return MOE_ERR_CUDA;
  g_last_launches = 0;
  return MOE_OK;
}

}  // namespace

cudaError_t current_context_id(unsigned long long* id) {
  static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 4000, cudaEnableDefault, &q) ==
            cudaSuccess && q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess && q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
  });
  if (get_current == nullptr || get_id == nullptr) return cudaErrorNotSupported;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS) return cudaErrorDeviceUninitialized;
  if (ctx == nullptr) {
    // no context yet on this thread: cudaSetDevice makes the device's primary context
    // current (initialising it), as every later runtime call would
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaSetDevice(dev);
    if (e != cudaSuccess) return e;
    if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return cudaErrorDeviceUninitialized;
  }
  return get_id(ctx, id) == CUDA_SUCCESS ? cudaSuccess : cudaErrorDeviceUninitialized;
}

moe_status check_config_host(const moe_config* cfg) { return check_config(cfg); }
int64_t capacity_host(const moe_config* cfg) { return capacity_of(cfg); }
void set_last_launch_count(int32_t n) { g_last_launches = n; }

}  // namespace moe

using namespace moe;

extern "C" {

const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_DEVICE: return "device error bits set";
  }
  return "unknown status";
}

int64_t moe_capacity(const moe_config* cfg) {
  if (check_config(cfg) == MOE_ERR_INVALID_ARG) return -2;
  return capacity_of(cfg);
}

size_t moe_workspace_size(const moe_config* cfg) {
  if (check_config(cfg) != MOE_OK) return 0;
  return layout(cfg).steps;
}

size_t moe_forward_workspace_size(const moe_config* cfg) {
  if (check_config(cfg) != MOE_OK) return 0;
  return layout(cfg).forward;
}

moe_status moe_route(const moe_config* cfg, const void* x, const void* w_gate, const void* w_noise,
                     const float* noise, const float* logit_bias, int32_t* topk_idx,
                     float* topk_gate, float* importance, float* load, uint8_t* near_tie, void* ws,
                     moe_stream_t stream) {
  moe_status st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (cfg->T == 0) return empty_batch(cfg, nullptr, nullptr, importance, load, stream);
  st = check_route_args(cfg, x, w_gate, w_noise, noise, topk_idx, topk_gate, importance, load,
                          ws);
  if (st != MOE_OK) return st;
  Ctx ctx(ws, stream);
  if (!ctx.ok) return MOE_ERR_CUDA;
  st = do_route(cfg, layout(cfg), x, w_gate, w_noise, noise, logit_bias, topk_idx, topk_gate,
                importance, load, near_tie, ws, ctx);
  return st == MOE_OK ? ctx.finish(cudaSuccess) : st;
}

moe_status moe_permute(const moe_config* cfg, const int32_t* topk_idx, const void* x,
                       int32_t* counts, int32_t* offsets, int32_t* perm_src, int32_t* slot_pos,
                       void* x_perm, void* ws, moe_stream_t stream) {
  moe_status st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (!counts || !offsets) return MOE_ERR_INVALID_ARG;
  if (cfg->T == 0) return empty_batch(cfg, counts, offsets, nullptr, nullptr, stream);
  if (!topk_idx || !perm_src || !slot_pos || !ws || (x_perm && !x)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(ws) || (x_perm && (!aligned16(x) || !aligned16(x_perm)))) return MOE_ERR_INVALID_ARG;
  Ctx ctx(ws, stream);
  if (!ctx.ok) return MOE_ERR_CUDA;
  st = do_permute(cfg, layout(cfg), topk_idx, x, counts, offsets, perm_src, slot_pos, x_perm, ws, ctx);
  return st == MOE_OK ? ctx.finish(cudaSuccess) : st;
}

moe_status moe_expert_ffn(const moe_config* cfg, const void* x_perm, const int32_t* offsets,
                          const void* w1, const void* w2, void* h, void* y_perm, void* ws,
                          moe_stream_t stream) {
  moe_status st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (cfg->T == 0) {
    g_last_launches = 0;
    return MOE_OK;
  }
  if (!x_perm || !offsets || !w1 || !w2 || !h || !y_perm || !ws) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x_perm) || !aligned16(w1) || !aligned16(w2) || !aligned16(h) ||
      !aligned16(y_perm) || !aligned16(ws))
    return MOE_ERR_INVALID_ARG;
  Ctx ctx(ws, stream);
  if (!ctx.ok) return MOE_ERR_CUDA;
  st = do_ffn(cfg, x_perm, offsets, w1, w2, h, y_perm, ctx);
  return st == MOE_OK ? ctx.finish(cudaSuccess) : st;
}

moe_status moe_expert_ffn_grouped(const moe_config* cfg, const void* x_rows, int64_t rows_cap,
                                  const int32_t* offsets, int32_t groups, const void* w1,
                                  const void* w2, void* h, void* y_rows, void* ws,
                                  moe_stream_t stream) {
  moe_status st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (cfg->dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
  if (rows_cap < 0 || groups <= 0) return MOE_ERR_INVALID_ARG;
  if (groups > 1024 || rows_cap >= (int64_t{1} << 31)) return MOE_ERR_UNSUPPORTED;
  if (rows_cap == 0) {
    g_last_launches = 0;
    return MOE_OK;
  }
  if (!x_rows || !offsets || !w1 || !w2 || !h || !y_rows || !ws) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x_rows) || !aligned16(w1) || !aligned16(w2) || !aligned16(h) ||
      !aligned16(y_rows) || !aligned16(ws))
    return MOE_ERR_INVALID_ARG;
  Ctx ctx(ws, stream);
  if (!ctx.ok) return MOE_ERR_CUDA;
  FfnProblem p;
  p.x_rows = rows_cap;
  p.rows_cap = rows_cap;
  p.d = cfg->d_model;
  p.f = cfg->d_ff;
  p.E = groups;
  p.w_count = cfg->E;
  p.act = cfg->act == MOE_ACT_GELU ? 2 : 1;
  p.hidden_f16 = cfg->hidden_f16;
  p.x_perm = x_rows;
  p.offsets = offsets;
  p.w1 = w1;
  p.w2 = w2;
  p.h = h;
  p.y_perm = y_rows;
  const cudaError_t e = launch_ffn_bf16(p, ctx.lc);
  return ctx.finish(e);
}

moe_status moe_expert_ffn_gather(const moe_config* cfg, const void* x, const int32_t* perm_src,
                                 const int32_t* offsets, const void* w1, const void* w2, void* h,
                                 void* y_perm, void* ws, moe_stream_t stream) {
  moe_status st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (cfg->T == 0) {
    g_last_launches = 0;
    return MOE_OK;
  }
  if (!x || !perm_src || !offsets || !w1 || !w2 || !h || !y_perm || !ws) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w1) || !aligned16(w2) || !aligned16(h) || !aligned16(y_perm) ||
      !aligned16(ws))
    return MOE_ERR_INVALID_ARG;
  Ctx ctx(ws, stream);
  if (!ctx.ok) return MOE_ERR_CUDA;
  st = do_ffn(cfg, nullptr, offsets, w1, w2, h, y_perm, ctx, x, perm_src);
  return st == MOE_OK ? ctx.finish(cudaSuccess) : st;
}

moe_status moe_combine(const moe_config* cfg, const void* y_perm, const int32_t* slot_pos,
                       const float* topk_gate, void* y, void* ws, moe_stream_t stream) {
  moe_status st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (cfg->T == 0) {
    g_last_launches = 0;
    return MOE_OK;
  }
  if (!y_perm || !slot_pos || !topk_gate || !y || !ws) return MOE_ERR_INVALID_ARG;
  if (!aligned16(y_perm) || !aligned16(y) || !aligned16(ws)) return MOE_ERR_INVALID_ARG;
  Ctx ctx(ws, stream);
  if (!ctx.ok) return MOE_ERR_CUDA;
  st = do_combine(cfg, y_perm, slot_pos, topk_gate, y, ctx);
  return st == MOE_OK ? ctx.finish(cudaSuccess) : st;
}

moe_status moe_expert_ffn_combine(const moe_config* cfg, const void* x_perm,
                                  const int32_t* offsets, const int32_t* perm_src,
                                  const int32_t* slot_pos, const float* topk_gate,
                                  const void* w1, const void* w2, void* h, void* y, void* ws,
                                  moe_stream_t stream) {
  moe_status st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (!fused_combine(cfg)) return MOE_ERR_UNSUPPORTED;
  if (cfg->T == 0) {
    g_last_launches = 0;
    return MOE_OK;
  }
  if (!x_perm || !offsets || !perm_src || !slot_pos || !topk_gate || !w1 || !w2 || !h || !y || !ws)
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(x_perm) || !aligned16(w1) || !aligned16(w2) || !aligned16(h) || !aligned16(y) ||
      !aligned16(ws))
    return MOE_ERR_INVALID_ARG;
  Ctx ctx(ws, stream);
  if (!ctx.ok) return MOE_ERR_CUDA;
  st = do_ffn_combine(cfg, x_perm, offsets, perm_src, slot_pos, topk_gate, w1, w2, h, y, ctx);
  return st == MOE_OK ? ctx.finish(cudaSuccess) : st;
}

moe_status moe_expert_ffn_combine_gather(const moe_config* cfg, const void* x,
                                         const int32_t* offsets, const int32_t* perm_src,
                                         const int32_t* slot_pos, const float* topk_gate,
                                         const void* w1, const void* w2, void* h, void* y,
                                         void* ws, moe_stream_t stream) {
  moe_status st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (!fused_combine(cfg)) return MOE_ERR_UNSUPPORTED;
  if (cfg->T == 0) {
    g_last_launches = 0;
    return MOE_OK;
  }
  if (!x || !offsets || !perm_src || !slot_pos || !topk_gate || !w1 || !w2 || !h || !y || !ws)
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w1) || !aligned16(w2) || !aligned16(h) || !aligned16(y) ||
      !aligned16(ws))
    return MOE_ERR_INVALID_ARG;
  Ctx ctx(ws, stream);
  if (!ctx.ok) return MOE_ERR_CUDA;
  st = do_ffn_combine(cfg, nullptr, offsets, perm_src, slot_pos, topk_gate, w1, w2, h, y, ctx, x,
                      true);
  return st == MOE_OK ? ctx.finish(cudaSuccess) : st;
}

moe_status moe_forward(const moe_config* cfg, const void* x, const void* w_gate, const void* w_noise,
                       const float* noise, const float* logit_bias, const void* w1, const void* w2,
                       void* y, int32_t* topk_idx, float* topk_gate, int32_t* counts,
                       float* importance, float* load, uint8_t* near_tie, void* ws,
                       moe_stream_t stream) {
  moe_status st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (!counts) return MOE_ERR_INVALID_ARG;
  if (cfg->T == 0) return empty_batch(cfg, counts, nullptr, importance, load, stream);
  st = check_route_args(cfg, x, w_gate, w_noise, noise, topk_idx, topk_gate, importance, load,
                          ws);
  if (st != MOE_OK) return st;
  if (!w1 || !w2 || !y) return MOE_ERR_INVALID_ARG;
  if (!aligned16(w1) || !aligned16(w2) || !aligned16(y)) return MOE_ERR_INVALID_ARG;
  Ctx ctx(ws, stream);
  if (!ctx.ok) return MOE_ERR_CUDA;
  const Layout L = layout(cfg);
  uint8_t* w = static_cast<uint8_t*>(ws);
  int32_t* offsets = reinterpret_cast<int32_t*>(w + L.offsets);
  int32_t* slot_pos = reinterpret_cast<int32_t*>(w + L.slot_pos);
  int32_t* perm_src = reinterpret_cast<int32_t*>(w + L.perm_src);
  void* x_perm = w + L.x_perm;
  void* h = w + L.h;
  void* y_perm = w + L.y_perm;
  st = do_route(cfg, L, x, w_gate, w_noise, noise, logit_bias, topk_idx, topk_gate, importance, load,
                near_tie, ws, ctx);
  if (st != MOE_OK) return st;
  // the kept rows are copied into x_perm once and read by tiled TMA loads: measured
  // faster than gathering them inside the up-projection (tile::gather4)
  st = do_permute(cfg, L, topk_idx, x, counts, offsets, perm_src, slot_pos, x_perm, ws, ctx);
  if (st != MOE_OK) return st;
  // k = 1: the down-projection stores y itself.  k = 2 takes the two steps: its fused form
  // (in-memory adds onto a zeroed y) measured no faster on zipf and 3% slower on gshard
  if (cfg->k == 1 && fused_combine(cfg)) {
    st = do_ffn_combine(cfg, x_perm, offsets, perm_src, slot_pos, topk_gate, w1, w2, h, y, ctx);
    if (st != MOE_OK) return st;
    return ctx.finish(cudaSuccess);
  }
  st = do_ffn(cfg, x_perm, offsets, w1, w2, h, y_perm, ctx);
  if (st != MOE_OK) return st;
  st = do_combine(cfg, y_perm, slot_pos, topk_gate, y, ctx);
  if (st != MOE_OK) return st;
  return ctx.finish(cudaSuccess);
}

size_t moe_train_state_size(const moe_config* cfg) {
  if (check_train_config(cfg) != MOE_OK) return 0;
  return train_layout(cfg).total;
}

size_t moe_backward_workspace_size(const moe_config* cfg) {
  if (check_train_config(cfg) != MOE_OK) return 0;
  return backward_layout(cfg, layout(cfg).steps).total;
}

moe_status moe_forward_train(const moe_config* cfg, const void* x, const void* w_gate,
                             const void* w_noise, const float* noise, const float* logit_bias,
                             const void* w1, const void* w2, void* y, int32_t* topk_idx,
                             float* topk_gate, int32_t* counts, float* importance, float* load,
                             uint8_t* near_tie, void* state, void* ws, moe_stream_t stream) {
  moe_status st = check_train_config(cfg);
  if (st != MOE_OK) return st;
  if (!counts || !state) return MOE_ERR_INVALID_ARG;
  if (cfg->T == 0) return empty_batch(cfg, counts, nullptr, importance, load, stream);
  st = check_route_args(cfg, x, w_gate, w_noise, noise, topk_idx, topk_gate, importance, load, ws);
  if (st != MOE_OK) return st;
  if (!w1 || !w2 || !y || !aligned16(w1) || !aligned16(w2) || !aligned16(y) || !aligned16(state))
    return MOE_ERR_INVALID_ARG;
  Ctx ctx(ws, stream);
  if (!ctx.ok) return MOE_ERR_CUDA;
  const Layout L = layout(cfg);
  const TrainLayout S = train_layout(cfg);
  uint8_t* sb = static_cast<uint8_t*>(state);
  int32_t* offsets = reinterpret_cast<int32_t*>(sb + S.offsets);
  int32_t* slot_pos = reinterpret_cast<int32_t*>(sb + S.slot_pos);
  int32_t* perm_src = reinterpret_cast<int32_t*>(sb + S.perm_src);
  void* x_perm = sb + S.x_perm;
  void* u = sb + S.u;
  void* h = sb + S.h;
  void* y_perm = sb + S.y_perm;
  st = do_route(cfg, L, x, w_gate, w_noise, noise, logit_bias, topk_idx, topk_gate, importance, load,
                near_tie, ws, ctx, sb);
  if (st != MOE_OK) return st;
  st = do_permute(cfg, L, topk_idx, x, counts, offsets, perm_src, slot_pos, x_perm, ws, ctx);
  if (st != MOE_OK) return st;
  st = do_ffn(cfg, x_perm, offsets, w1, w2, h, y_perm, ctx, nullptr, nullptr, u);
  if (st != MOE_OK) return st;
  st = do_combine(cfg, y_perm, slot_pos, topk_gate, y, ctx);
  if (st != MOE_OK) return st;
  return ctx.finish(cudaSuccess);
}

moe_status moe_backward(const moe_config* cfg, const void* x, const void* w_gate,
                        const void* w_noise, const float* noise, const float* logit_bias,
                        const void* w1, const void* w2, const int32_t* topk_idx,
                        const float* topk_gate, const float* importance, const float* load,
                        const void* state, const float* dy, float w_importance, float w_load,
                        float* dx, float* dw_gate, float* dw_noise, float* dlogit_bias, float* dw1,
                        float* dw2, float* dgates, float* losses, void* ws, moe_stream_t stream) {
  moe_status st = check_train_config(cfg);
  if (st != MOE_OK) return st;
  const bool noisy = cfg->gating == MOE_GATE_NOISY_TOPK;
  if (!(w_importance == w_importance) || !(w_load == w_load)) return MOE_ERR_INVALID_ARG;
  if (w_importance != 0.0f && !importance) return MOE_ERR_INVALID_ARG;
  if (w_load != 0.0f && !(noisy && load && cfg->k < cfg->E)) return MOE_ERR_INVALID_ARG;
  if (!x || !w_gate || !w1 || !w2 || !topk_idx || !topk_gate || !state || !dy || !dx || !dw_gate ||
      !dw1 || !dw2 || !dgates || !ws)
    return MOE_ERR_INVALID_ARG;
  if (noisy && (!w_noise || !noise || !dw_noise)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w_gate) || !aligned16(w1) || !aligned16(w2) || !aligned16(state) ||
      !aligned16(dy) || !aligned16(dx) || !aligned16(dw1) || !aligned16(dw2) || !aligned16(ws) ||
      (noisy && !aligned16(w_noise)))
    return MOE_ERR_INVALID_ARG;
  if (cfg->T == 0) {
    g_last_launches = 0;
    return MOE_OK;
  }
  Ctx ctx(ws, stream);
  if (!ctx.ok) return MOE_ERR_CUDA;
  const Layout L = layout(cfg);
  const TrainLayout S = train_layout(cfg);
  const BackwardLayout B = backward_layout(cfg, L.steps);
  const uint8_t* sb = static_cast<const uint8_t*>(state);
  uint8_t* w = static_cast<uint8_t*>(ws);
  BackwardProblem p;
  p.T = cfg->T;
  p.d = cfg->d_model;
  p.f = cfg->d_ff;
  p.E = cfg->E;
  p.k = cfg->k;
  p.act = cfg->act == MOE_ACT_GELU ? 2 : 1;
  p.noisy = noisy;
  p.renorm = cfg->renorm != 0;
  p.hidden_f16 = cfg->hidden_f16;
  p.w_importance = w_importance;
  p.w_load = w_load;
  p.x = x;
  p.w_gate = w_gate;
  p.w_noise = w_noise;
  p.noise = noise;
  p.bias = logit_bias;
  p.w1 = w1;
  p.w2 = w2;
  p.topk_idx = topk_idx;
  p.topk_gate = topk_gate;
  p.importance = importance;
  p.load = load;
  p.offsets = reinterpret_cast<const int32_t*>(sb + S.offsets);
  p.slot_pos = reinterpret_cast<const int32_t*>(sb + S.slot_pos);
  p.x_perm = sb + S.x_perm;
  p.u = sb + S.u;
  p.h = sb + S.h;
  p.y_perm = reinterpret_cast<const float*>(sb + S.y_perm);
  p.dy = dy;
  p.dx = dx;
  p.dw_gate = dw_gate;
  p.dw_noise = dw_noise;
  p.dbias = dlogit_bias;
  p.dw1 = dw1;
  p.dw2 = dw2;
  p.dgate = dgates;
  p.losses = losses;
  p.poff = reinterpret_cast<int32_t*>(w + B.poff);
  p.d_o = w + B.d_o;
  p.du = w + B.du;
  p.dx_perm = reinterpret_cast<float*>(w + B.dx_perm);
  p.lg = reinterpret_cast<const float*>(sb + S.lg);
  p.sw = noisy ? reinterpret_cast<const float*>(sb + S.sw) : nullptr;
  p.hw = noisy ? reinterpret_cast<const float*>(sb + S.hw) : nullptr;
  p.dl = reinterpret_cast<float*>(w + B.dl);
  p.dz = noisy ? p.dl + cfg->T * cfg->E : nullptr;
  p.dimp = reinterpret_cast<float*>(w + B.dimp);
  p.dload = reinterpret_cast<float*>(w + B.dload);
  p.part = reinterpret_cast<float*>(w + B.part);
  p.part_cap = B.part_cap;
  if (losses && cudaMemsetAsync(losses, 0, 2 * sizeof(float), ctx.lc.stream) != cudaSuccess)
    return MOE_ERR_CUDA;
  return ctx.finish(launch_backward(p, ctx.lc));
}

moe_status moe_get_error(void* ws, moe_stream_t stream, int32_t* device_error) {
  if (!ws) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int32_t v = 0;
  if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaMemcpy(&v, ws, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
  if (v != 0 && cudaMemset(ws, 0, 4) != cudaSuccess) return MOE_ERR_CUDA;
  if (device_error) *device_error = v;
  return v == 0 ? MOE_OK : MOE_ERR_DEVICE;
}

moe_status moe_bf16_to_f16(const void* src, void* dst, int64_t n, int32_t* n_inexact,
                           moe_stream_t stream) {
  if (n < 0 || (n > 0 && (!src || !dst))) return MOE_ERR_INVALID_ARG;
  if (n == 0) {
    g_last_launches = 0;
    return MOE_OK;
  }
  Ctx ctx(nullptr, stream);
  if (!ctx.ok) return MOE_ERR_CUDA;
  return ctx.finish(launch_bf16_to_f16(src, dst, n, n_inexact, ctx.lc));
}

moe_status moe_wait_timeout_check(void* ws, moe_stream_t stream) {
  if (!ws || !aligned16(ws)) return MOE_ERR_INVALID_ARG;
  Ctx ctx(ws, stream);
  if (!ctx.ok) return MOE_ERR_CUDA;
  // the barrier counters are words 2 and 3 of the error block, as for moe_permute
  int32_t* sync = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(ws) + 8);
  return ctx.finish(launch_wait_timeout_check(sync, ctx.lc.err, ctx.lc));
}

int32_t moe_last_launch_count(void) { return g_last_launches; }

}  // extern "C"
