// C-ABI entry points: host-side validation, regime choice and launches.
// Nothing here synchronises with the device or allocates memory.
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdio>
#include <cstring>

#include "../../include/lora_delta.h"
#include "kernels.h"
#include "sgmv.h"

namespace {

thread_local char g_last_error[512] = "";

lora_status fail(lora_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return st;
}

lora_status ok() {
  g_last_error[0] = '\0';
  return LORA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

lora_status cuda_fail(cudaError_t err, const char* what, const char* why) {
  if (why != nullptr) return fail(LORA_ERR_UNSUPPORTED, "%s: %s", what, why);
  return fail(LORA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(err));
}

// Checks shared by every linear / embedding entry point.  Fills slice_off.
lora_status check_common(const char* op, int32_t T, int32_t in_features, int32_t slots,
                         int32_t R, int32_t num_slices, const int32_t* out_slices,
                         bool need_out, int* slice_off, int* out_total) {
  if (T < 0) return fail(LORA_ERR_INVALID, "%s: T = %d < 0", op, T);
  if (slots < 0) return fail(LORA_ERR_INVALID, "%s: slots = %d < 0", op, slots);
  if (slots > LORA_MAX_SLOTS)
    return fail(LORA_ERR_UNSUPPORTED, "%s: slots = %d > %d", op, slots, LORA_MAX_SLOTS);
  if (R <= 0 || R % 8 != 0)
    return fail(LORA_ERR_INVALID, "%s: R = %d must be a positive multiple of 8", op, R);
  if (in_features <= 0 || in_features % 8 != 0)
    return fail(LORA_ERR_INVALID, "%s: in_features = %d must be a positive multiple of 8", op,
                in_features);
  if (num_slices < 1 || num_slices > LORA_MAX_SLICES)
    return fail(LORA_ERR_INVALID, "%s: num_slices = %d outside [1, %d]", op, num_slices,
                LORA_MAX_SLICES);
  slice_off[0] = 0;
  if (need_out) {
    if (out_slices == nullptr) return fail(LORA_ERR_INVALID, "%s: out_slices is NULL", op);
    long long tot = 0;
    for (int i = 0; i < num_slices; ++i) {
      if (out_slices[i] <= 0 || out_slices[i] % 8 != 0)
        return fail(LORA_ERR_INVALID, "%s: out_slices[%d] = %d must be a positive multiple of 8",
                    op, i, out_slices[i]);
      tot += out_slices[i];
      if (tot > (1 << 30)) return fail(LORA_ERR_UNSUPPORTED, "%s: out too large", op);
      slice_off[i + 1] = (int)tot;
    }
    *out_total = (int)tot;
  } else {
    for (int i = 0; i < num_slices; ++i) slice_off[i + 1] = 0;
    *out_total = 0;
  }
  for (int i = num_slices + 1; i <= LORA_MAX_SLICES; ++i) slice_off[i] = slice_off[num_slices];
  return LORA_OK;
}

lora_status check_ptrs(const char* op, std::initializer_list<std::pair<const void*, const char*>> p16,
                       std::initializer_list<std::pair<const void*, const char*>> p4) {
  for (auto& q : p16) {
    if (q.first == nullptr) return fail(LORA_ERR_INVALID, "%s: %s is NULL", op, q.second);
    if (!aligned16(q.first))
      return fail(LORA_ERR_INVALID, "%s: %s is not 16-byte aligned", op, q.second);
  }
  for (auto& q : p4) {
    if (q.first == nullptr) return fail(LORA_ERR_INVALID, "%s: %s is NULL", op, q.second);
    if (!aligned4(q.first))
      return fail(LORA_ERR_INVALID, "%s: %s is not 4-byte aligned", op, q.second);
  }
  return LORA_OK;
}

bool bgmv_fits(int S, int R) { return S * lora::round_up_i(R, 16) <= lora::kMaxSRp; }

// The fused apply's shapes AUTO streams (given the workspace): measured on
// the B200 against SGMV and BGMV with S*R <= 64, the short-segment shrink and
// the streamed expand are ahead from T = 512 (BGMV ahead below) up to
// T * in_features = 2^25 and T * out = 2^26 (SGMV ahead beyond), and at
// T = 16384 SGMV is ahead again.
constexpr int kStreamLinearMinT = 512;
constexpr int kStreamLinearMaxT = 8192;
constexpr long long kStreamLinearMaxIn = 1LL << 25;    // T * in_features
constexpr long long kStreamLinearMaxOut = 1LL << 26;   // T * out

bool stream_linear_fits(int T, int in_features, int out, int S, int R) {
  return lora::stream_supported(R) && lora::group_shrink_supported(S, R, in_features) &&
         T >= kStreamLinearMinT && T <= kStreamLinearMaxT &&
         (long long)T * in_features <= kStreamLinearMaxIn &&
         (long long)T * out <= kStreamLinearMaxOut;
}

int resolve(int regime, int op, int T, int slots, int R, int S, int in_features = 1 << 30) {
  if (regime == LORA_REGIME_BGMV || regime == LORA_REGIME_SGMV) return regime;
  if (regime == LORA_REGIME_BGMV_SPLIT)
    return op == LORA_OP_APPLY_LINEAR ? LORA_REGIME_BGMV_SPLIT : LORA_REGIME_BGMV;
  if (regime == LORA_REGIME_STREAM)
    return (op == LORA_OP_APPLY_EMBEDDING || op == LORA_OP_APPLY_LINEAR) ? LORA_REGIME_STREAM
                                                                         : LORA_REGIME_BGMV;
  // the embedding: stream the output rows through shared memory
  if (op == LORA_OP_APPLY_EMBEDDING && lora::stream_supported(R)) return LORA_REGIME_STREAM;
  const bool needs_shrink = (op == LORA_OP_SHRINK || op == LORA_OP_APPLY_LINEAR);
  // Many tokens per slot on average: tensor-core tiles over slot segments.
  if (lora::sgmv_supported(S, R) && slots > 0 && (long long)T >= 64LL * slots && T >= 1024 &&
      (!needs_shrink || in_features >= 64))
    return LORA_REGIME_SGMV;
  return LORA_REGIME_BGMV;
}

// Workspace bytes lora_apply_linear needs in regime `reg` (0: none).  SGMV:
// the counter header (which it leaves alone), then the partial h buffers of
// the split shrink.  BGMV_SPLIT: its counters and partials.  STREAM: the
// counter header (which it leaves alone), then the partial h of every chunk
// of the input features (at most eight).  BGMV: none.
size_t apply_linear_need(int reg, int T, int in_features, int slots, int R, int S, int out) {
  if (T <= 0 || R <= 0 || S <= 0) return 0;
  if (reg == LORA_REGIME_SGMV) return lora::kWsCounterBytes + lora::sgmv_workspace_bytes(T, R, S);
  if (reg == LORA_REGIME_STREAM)
    return lora::kWsCounterBytes +
           (size_t)lora::group_shrink_chunks(in_features) * T * S * R * sizeof(float);
  if (reg == LORA_REGIME_BGMV_SPLIT && lora::split_eligible(T, in_features, slots, R, S, out))
    return lora::split_workspace_bytes(T, slots, R, S);
  return 0;
}

// Workspace of the grouped expert fold: token_order [rows_cap], the group
// tables (seg_lo, seg_hi, g_rank, g_scal; kMoeMaxGroups each), then the
// partial h buffers (the short-segment shrink's eight, or the SGMV shrink's
// four).  0 when the shapes are not the SGMV kernels'.
size_t expert_group_need(int rows_cap, int R, int S) {
  if (rows_cap <= 0 || !lora::sgmv_supported(S, R)) return 0;
  const size_t tok = ((size_t)rows_cap * 4 + 255) / 256 * 256;
  const size_t tables = (size_t)4 * lora::kMoeMaxGroups * 4;
  const size_t parts = (size_t)lora::kGsMaxParts * rows_cap * R * S * sizeof(float);
  const size_t sgmv = lora::sgmv_workspace_bytes(rows_cap, R, S);
  return tok + tables + (parts > sgmv ? parts : sgmv);
}

// lora_apply_linear's regime: resolve()'s, except that AUTO streams the
// shapes stream_linear_fits() takes when ws_bytes holds the STREAM workspace.
int resolve_linear(int regime, int T, int slots, int R, int S, int in_features, int out,
                   size_t ws_bytes) {
  const int reg = resolve(regime, LORA_OP_APPLY_LINEAR, T, slots, R, S, in_features);
  if (regime == LORA_REGIME_AUTO && stream_linear_fits(T, in_features, out, S, R) &&
      ws_bytes >= apply_linear_need(LORA_REGIME_STREAM, T, in_features, slots, R, S, out))
    return LORA_REGIME_STREAM;
  return reg;
}

int linear_items_bound(int T, int slots, int tile) {
  const long long b = (long long)slots + ((long long)T + tile - 1) / tile;
  return (int)(b > (1LL << 30) ? (1LL << 30) : b);
}

}  // namespace

namespace lora {
// Lets other entry points of the library report through lora_last_error().
void set_last_error(const char* msg) { snprintf(g_last_error, sizeof(g_last_error), "%s", msg); }
size_t apply_linear_workspace(int regime, int T, int in_features, int slots, int R, int S,
                              int out, size_t ws_bytes) {
  const int reg = resolve_linear(regime, T, slots, R, S, in_features, out, ws_bytes);
  return apply_linear_need(reg, T, in_features, slots, R, S, out);
}
}  // namespace lora

extern "C" {

const char* lora_status_string(lora_status status) {
  switch (status) {
    case LORA_OK: return "LORA_OK";
    case LORA_ERR_INVALID: return "LORA_ERR_INVALID";
    case LORA_ERR_UNSUPPORTED: return "LORA_ERR_UNSUPPORTED";
    case LORA_ERR_WORKSPACE: return "LORA_ERR_WORKSPACE";
    case LORA_ERR_CUDA: return "LORA_ERR_CUDA";
  }
  return "LORA_ERR_UNKNOWN";
}

const char* lora_last_error(void) { return g_last_error; }

int32_t lora_set_launch_overlap(int32_t enable) { return lora::bgmv_set_overlap(enable); }

const char* lora_version(void) { return "lora_delta 0.1.0 sm_100a"; }

int32_t lora_resolve_regime(int32_t op, int32_t T, int32_t slots, int32_t R, int32_t num_slices) {
  if (op == LORA_OP_EXPERT_APPLY) return LORA_REGIME_BGMV;
  return resolve(LORA_REGIME_AUTO, op, T, slots, R, num_slices);
}

int32_t lora_plan_tile(int32_t op, int32_t regime) {
  if (op == LORA_OP_EXPERT_APPLY) return lora::kTT;
  if ((op == LORA_OP_APPLY_EMBEDDING || op == LORA_OP_APPLY_LINEAR) &&
      regime == LORA_REGIME_STREAM)
    return lora::kStRows;
  if (regime == LORA_REGIME_SGMV) return lora::kSgmvTileM;
  if (op == LORA_OP_APPLY_LINEAR) return lora::kFusedTile;
  return lora::kTT;
}

size_t lora_workspace_bytes(int32_t op, int32_t T, int32_t slots, int32_t R, int32_t num_slices,
                            int32_t regime) {
  if (op == LORA_OP_EXPERT_APPLY) {
    // the grouped (tensor-core) fold; BGMV asks for the per-chunk kernel
    if (regime == LORA_REGIME_BGMV || T <= 0 || R <= 0 || num_slices <= 0) return 0;
    return expert_group_need(T, R, num_slices);
  }
  if (op != LORA_OP_APPLY_LINEAR || T <= 0 || R <= 0 || num_slices <= 0) return 0;
  const int reg = resolve(regime, op, T, slots, R, num_slices);
  // in_features and out are not known here: size for the largest the split
  // and streamed kernels take (they refuse larger ones)
  if (reg == LORA_REGIME_STREAM)
    return apply_linear_need(reg, T, lora::kGsMaxIn, slots, R, num_slices, 0);
  size_t need = apply_linear_need(reg, T, lora::kSpMaxIn, slots, R, num_slices, lora::kSpMaxOut);
  if (regime == LORA_REGIME_AUTO) {
    // AUTO streams these shapes when in_features is small enough (and is
    // given the workspace): room for the largest such in_features
    long long in_max = kStreamLinearMaxIn / T;
    in_max = (in_max < lora::kGsMaxIn ? in_max : lora::kGsMaxIn) / 8 * 8;
    if (in_max >= 8 && stream_linear_fits(T, (int)in_max, 8, num_slices, R)) {
      const size_t sneed =
          apply_linear_need(LORA_REGIME_STREAM, T, (int)in_max, slots, R, num_slices, 0);
      need = sneed > need ? sneed : need;
    }
  }
  return need;
}

uint64_t lora_set_wait_limit_ns(uint64_t ns) { return lora::set_wait_limit_ns(ns); }

lora_status lora_shrink(const void* x, float* h, const void* a, const int32_t* ranks,
                        const int32_t* token_order, const int32_t* slot_indptr, int32_t T,
                        int32_t in_features, int32_t slots, int32_t R, int32_t num_slices,
                        int32_t regime, uint32_t* err_flags, void* stream) {
  const char* op = "lora_shrink";
  lora::BgmvParams p = {};
  int out = 0;
  lora_status st = check_common(op, T, in_features, slots, R, num_slices, nullptr, false,
                                p.slice_off, &out);
  if (st != LORA_OK) return st;
  if (T == 0 || slots == 0) return ok();
  st = check_ptrs(op, {{x, "x"}, {h, "h"}, {a, "a"}},
                  {{ranks, "ranks"}, {token_order, "token_order"}, {slot_indptr, "slot_indptr"}});
  if (st != LORA_OK) return st;
  if (err_flags != nullptr && !aligned4(err_flags))
    return fail(LORA_ERR_INVALID, "%s: err_flags is not 4-byte aligned", op);
  const int reg = resolve(regime, LORA_OP_SHRINK, T, slots, R, num_slices, in_features);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (reg == LORA_REGIME_SGMV) {
    if (!lora::sgmv_supported(num_slices, R))
      return fail(LORA_ERR_UNSUPPORTED, "%s: %s", op, lora::kSgmvShapeRule);
    const char* why = nullptr;
    cudaError_t err = lora::sgmv_shrink_launch(x, a, h, ranks, token_order, slot_indptr, T,
                                               in_features, slots, R, num_slices, err_flags, s,
                                               &why, 1, nullptr);
    if (err != cudaSuccess) return cuda_fail(err, op, why);
    return ok();
  }
  if (!bgmv_fits(num_slices, R))
    return fail(LORA_ERR_UNSUPPORTED, "%s: num_slices*roundup(R,16) = %d > %d", op,
                num_slices * lora::round_up_i(R, 16), lora::kMaxSRp);
  p.x = x; p.h = h; p.a = a; p.ranks = ranks; p.token_order = token_order;
  p.slot_indptr = slot_indptr; p.flags = err_flags; p.T = T; p.in = in_features;
  p.slots = slots; p.R = R; p.S = num_slices; p.out = 0;
  const char* why = nullptr;
  cudaError_t err = lora::bgmv_launch(lora::kModeShrink, p, linear_items_bound(T, slots, lora::kTT),
                                      s, &why);
  if (err != cudaSuccess) return cuda_fail(err, op, why);
  return ok();
}

lora_status lora_expand(void* y, const float* h, const void* b, const int32_t* ranks,
                        const float* scalings, const int32_t* token_order,
                        const int32_t* slot_indptr, int32_t T, int32_t slots, int32_t R,
                        const int32_t* out_slices, int32_t num_slices, int32_t regime,
                        uint32_t* err_flags, void* stream) {
  const char* op = "lora_expand";
  lora::BgmvParams p = {};
  int out = 0;
  lora_status st =
      check_common(op, T, 8, slots, R, num_slices, out_slices, true, p.slice_off, &out);
  if (st != LORA_OK) return st;
  if (T == 0 || slots == 0) return ok();
  st = check_ptrs(op, {{y, "y"}, {h, "h"}, {b, "b"}},
                  {{ranks, "ranks"}, {scalings, "scalings"}, {token_order, "token_order"},
                   {slot_indptr, "slot_indptr"}});
  if (st != LORA_OK) return st;
  if (err_flags != nullptr && !aligned4(err_flags))
    return fail(LORA_ERR_INVALID, "%s: err_flags is not 4-byte aligned", op);
  const int reg = resolve(regime, LORA_OP_EXPAND, T, slots, R, num_slices);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (reg == LORA_REGIME_SGMV) {
    if (!lora::sgmv_supported(num_slices, R))
      return fail(LORA_ERR_UNSUPPORTED, "%s: %s", op, lora::kSgmvShapeRule);
    const char* why = nullptr;
    cudaError_t err = lora::sgmv_expand_launch(y, h, 1, nullptr, nullptr, b, ranks, scalings,
                                               token_order, slot_indptr, T, 0, slots, R,
                                               num_slices, p.slice_off, out, err_flags, s, &why);
    if (err != cudaSuccess) return cuda_fail(err, op, why);
    return ok();
  }
  if (!bgmv_fits(num_slices, R))
    return fail(LORA_ERR_UNSUPPORTED, "%s: num_slices*roundup(R,16) = %d > %d", op,
                num_slices * lora::round_up_i(R, 16), lora::kMaxSRp);
  p.y = y; p.h = const_cast<float*>(h); p.b = b; p.ranks = ranks; p.scalings = scalings;
  p.token_order = token_order; p.slot_indptr = slot_indptr; p.flags = err_flags; p.T = T;
  p.in = 8; p.slots = slots; p.R = R; p.S = num_slices; p.out = out;
  const char* why = nullptr;
  cudaError_t err = lora::bgmv_launch(lora::kModeExpand, p, linear_items_bound(T, slots, lora::kTT),
                                      s, &why);
  if (err != cudaSuccess) return cuda_fail(err, op, why);
  return ok();
}

}  // extern "C"

namespace {

// The fused shrink + expand behind lora_apply_linear and lora_apply_router;
// `op` names the entry point in error messages.
lora_status apply_linear_impl(const char* op, const void* x, void* y, const void* a,
                              const void* b, const int32_t* ranks, const float* scalings,
                              const int32_t* token_order, const int32_t* slot_indptr, int32_t T,
                              int32_t in_features, int32_t slots, int32_t R,
                              const int32_t* out_slices, int32_t num_slices, int32_t regime,
                              void* workspace, size_t workspace_bytes, uint32_t* err_flags,
                              void* stream) {
  lora::BgmvParams p = {};
  int out = 0;
  lora_status st = check_common(op, T, in_features, slots, R, num_slices, out_slices, true,
                                p.slice_off, &out);
  if (st != LORA_OK) return st;
  if (T == 0 || slots == 0) return ok();
  st = check_ptrs(op, {{x, "x"}, {y, "y"}, {a, "a"}, {b, "b"}},
                  {{ranks, "ranks"}, {scalings, "scalings"}, {token_order, "token_order"},
                   {slot_indptr, "slot_indptr"}});
  if (st != LORA_OK) return st;
  if (err_flags != nullptr && !aligned4(err_flags))
    return fail(LORA_ERR_INVALID, "%s: err_flags is not 4-byte aligned", op);
  const int reg = resolve_linear(regime, T, slots, R, num_slices, in_features, out,
                                 workspace != nullptr ? workspace_bytes : 0);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (reg == LORA_REGIME_STREAM) {
    // short-segment shrink into per-chunk partial h, then the streamed expand
    if (!lora::stream_supported(R) || !lora::group_shrink_supported(num_slices, R, in_features))
      return fail(LORA_ERR_UNSUPPORTED,
                  "%s: the STREAM regime takes num_slices*R in {16, 32, 48, 64} and "
                  "in_features <= %d", op, lora::kGsMaxIn);
    const size_t need = apply_linear_need(reg, T, in_features, slots, R, num_slices, out);
    if (workspace == nullptr || workspace_bytes < need)
      return fail(LORA_ERR_WORKSPACE, "%s: workspace of %zu bytes needed, %zu given", op, need,
                  workspace == nullptr ? (size_t)0 : workspace_bytes);
    if (!aligned16(workspace))
      return fail(LORA_ERR_INVALID, "%s: workspace is not 16-byte aligned", op);
    float* hws = reinterpret_cast<float*>(static_cast<char*>(workspace) + lora::kWsCounterBytes);
    lora::StreamParams q = {};
    const char* why = nullptr;
    int ks = 1;
    cudaError_t err = lora::group_shrink_launch(x, a, hws, token_order, slot_indptr, nullptr,
                                                nullptr, ranks, scalings, T, in_features, slots,
                                                R, num_slices, &ks, s, true);
    if (err != cudaSuccess) return cuda_fail(err, op, nullptr);
    q.h = hws; q.h_split = (size_t)T * num_slices * R; q.ksplit = ks;
    q.y = y; q.b = b; q.ranks = ranks; q.scalings = scalings; q.token_order = token_order;
    q.slot_indptr = slot_indptr; q.flags = err_flags;
    q.T = T; q.vocab = 0; q.slots = slots; q.R = R; q.S = num_slices; q.out = out;
    for (int i = 0; i <= LORA_MAX_SLICES; ++i) q.slice_off[i] = p.slice_off[i];
    err = lora::stream_launch(q, s, true, &why);
    if (err != cudaSuccess) return cuda_fail(err, op, why);
    return ok();
  }
  if (reg == LORA_REGIME_SGMV) {
    if (!lora::sgmv_supported(num_slices, R))
      return fail(LORA_ERR_UNSUPPORTED, "%s: %s", op, lora::kSgmvShapeRule);
    const size_t need = apply_linear_need(reg, T, in_features, slots, R, num_slices, out);
    if (workspace == nullptr || workspace_bytes < need)
      return fail(LORA_ERR_WORKSPACE, "%s: workspace of %zu bytes needed, %zu given", op, need,
                  workspace == nullptr ? (size_t)0 : workspace_bytes);
    if (!aligned16(workspace))
      return fail(LORA_ERR_INVALID, "%s: workspace is not 16-byte aligned", op);
    float* hws = reinterpret_cast<float*>(static_cast<char*>(workspace) + lora::kWsCounterBytes);
    const char* why = nullptr;
    const int ks = lora::sgmv_shrink_splits(T, slots, in_features);
    cudaError_t err = lora::sgmv_shrink_launch(x, a, hws, ranks, token_order, slot_indptr, T,
                                               in_features, slots, R, num_slices, err_flags, s,
                                               &why, ks, scalings);
    if (err != cudaSuccess) return cuda_fail(err, op, why);
    err = lora::sgmv_expand_launch(y, hws, ks, nullptr, nullptr, b, ranks, scalings, token_order,
                                   slot_indptr, T, 0, slots, R, num_slices, p.slice_off, out,
                                   err_flags, s, &why);
    if (err != cudaSuccess) return cuda_fail(err, op, why);
    return ok();
  }
  if (!bgmv_fits(num_slices, R))
    return fail(LORA_ERR_UNSUPPORTED, "%s: num_slices*roundup(R,16) = %d > %d", op,
                num_slices * lora::round_up_i(R, 16), lora::kMaxSRp);
  if (reg == LORA_REGIME_BGMV_SPLIT) {
    // the split kernel: every SM shares the work, h partials through the workspace
    if (!lora::split_eligible(T, in_features, slots, R, num_slices, out))
      return fail(LORA_ERR_UNSUPPORTED,
                  "%s: BGMV_SPLIT takes T <= %d, slots <= %d, at most %d work items, "
                  "in_features <= %d, out <= %d and num_slices*roundup(R,16) <= %d",
                  op, lora::kSpMaxT, lora::kSpMaxSlots, lora::kSpMaxItems, lora::kSpMaxIn,
                  lora::kSpMaxOut, lora::kMaxSRp);
    const size_t need = lora::split_workspace_bytes(T, slots, R, num_slices);
    if (workspace == nullptr || workspace_bytes < need)
      return fail(LORA_ERR_WORKSPACE, "%s: workspace of %zu bytes needed, %zu given", op, need,
                  workspace == nullptr ? (size_t)0 : workspace_bytes);
    if (!aligned16(workspace))
      return fail(LORA_ERR_INVALID, "%s: workspace is not 16-byte aligned", op);
    lora::SplitParams q = {};
    q.x = x; q.y = y; q.a = a; q.b = b; q.ranks = ranks; q.scalings = scalings;
    q.token_order = token_order; q.slot_indptr = slot_indptr; q.flags = err_flags;
    const int cap = lora::split_item_cap(T, slots);
    q.cnt = static_cast<uint32_t*>(workspace);
    q.cons = q.cnt + cap;
    q.part = reinterpret_cast<float*>(static_cast<char*>(workspace) + lora::kWsCounterBytes);
    q.T = T; q.in = in_features; q.slots = slots; q.R = R; q.S = num_slices; q.out = out;
    q.item_cap = cap;
    for (int i = 0; i <= LORA_MAX_SLICES; ++i) q.slice_off[i] = p.slice_off[i];
    const char* why = nullptr;
    cudaError_t err = lora::split_launch(q, s, &why);
    if (err != cudaSuccess) return cuda_fail(err, op, why);
    return ok();
  }
  p.x = x; p.y = y; p.a = a; p.b = b; p.ranks = ranks; p.scalings = scalings;
  p.token_order = token_order; p.slot_indptr = slot_indptr; p.flags = err_flags; p.T = T;
  p.in = in_features; p.slots = slots; p.R = R; p.S = num_slices; p.out = out;
  const char* why = nullptr;
  cudaError_t err = lora::bgmv_launch(lora::kModeFused, p,
                                      linear_items_bound(T, slots, lora::kFusedTile), s, &why);
  if (err != cudaSuccess) return cuda_fail(err, op, why);
  return ok();
}

}  // namespace

extern "C" {

lora_status lora_apply_linear(const void* x, void* y, const void* a, const void* b,
                              const int32_t* ranks, const float* scalings,
                              const int32_t* token_order, const int32_t* slot_indptr, int32_t T,
                              int32_t in_features, int32_t slots, int32_t R,
                              const int32_t* out_slices, int32_t num_slices, int32_t regime,
                              void* workspace, size_t workspace_bytes, uint32_t* err_flags,
                              void* stream) {
  return apply_linear_impl("lora_apply_linear", x, y, a, b, ranks, scalings, token_order,
                           slot_indptr, T, in_features, slots, R, out_slices, num_slices, regime,
                           workspace, workspace_bytes, err_flags, stream);
}

lora_status lora_apply_router(const void* router_in, void* gate_logits, const void* a,
                              const void* b, const int32_t* ranks, const float* scalings,
                              const int32_t* token_order, const int32_t* slot_indptr, int32_t T,
                              int32_t hidden, int32_t slots, int32_t R, int32_t num_experts,
                              int32_t regime, void* workspace, size_t workspace_bytes,
                              uint32_t* err_flags, void* stream) {
  const char* op = "lora_apply_router";
  if (hidden <= 0 || hidden % 8 != 0)
    return fail(LORA_ERR_INVALID, "%s: hidden = %d must be a positive multiple of 8", op, hidden);
  if (num_experts <= 0 || num_experts % 8 != 0)
    return fail(LORA_ERR_INVALID, "%s: num_experts = %d must be a positive multiple of 8", op,
                num_experts);
  // one slice of num_experts logit columns: the routing logits are the output
  // of the router projection
  const int32_t out_slices[1] = {num_experts};
  return apply_linear_impl(op, router_in, gate_logits, a, b, ranks, scalings,
                           token_order, slot_indptr, T, hidden, slots, R, out_slices, 1, regime,
                           workspace, workspace_bytes, err_flags, stream);
}

lora_status lora_gather_shrink(const int32_t* ids, float* h, const void* a, const int32_t* ranks,
                               const int32_t* token_order, const int32_t* slot_indptr, int32_t T,
                               int32_t vocab, int32_t slots, int32_t R, int32_t num_slices,
                               uint32_t* err_flags, void* stream) {
  const char* op = "lora_gather_shrink";
  lora::BgmvParams p = {};
  int out = 0;
  if (vocab <= 0) return fail(LORA_ERR_INVALID, "%s: vocab = %d must be positive", op, vocab);
  lora_status st = check_common(op, T, 8, slots, R, num_slices, nullptr, false, p.slice_off, &out);
  if (st != LORA_OK) return st;
  if (T == 0 || slots == 0) return ok();
  st = check_ptrs(op, {{h, "h"}, {a, "a"}},
                  {{ids, "ids"}, {ranks, "ranks"}, {token_order, "token_order"},
                   {slot_indptr, "slot_indptr"}});
  if (st != LORA_OK) return st;
  if (err_flags != nullptr && !aligned4(err_flags))
    return fail(LORA_ERR_INVALID, "%s: err_flags is not 4-byte aligned", op);
  if (!bgmv_fits(num_slices, R))
    return fail(LORA_ERR_UNSUPPORTED, "%s: num_slices*roundup(R,16) = %d > %d", op,
                num_slices * lora::round_up_i(R, 16), lora::kMaxSRp);
  p.ids = ids; p.h = h; p.a = a; p.ranks = ranks; p.token_order = token_order;
  p.slot_indptr = slot_indptr; p.flags = err_flags; p.T = T; p.in = vocab; p.slots = slots;
  p.R = R; p.S = num_slices; p.out = 0;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const char* why = nullptr;
  cudaError_t err = lora::bgmv_launch(lora::kModeGather, p, linear_items_bound(T, slots, lora::kTT),
                                      s, &why);
  if (err != cudaSuccess) return cuda_fail(err, op, why);
  return ok();
}

lora_status lora_apply_embedding(const int32_t* ids, void* y, const void* a, const void* b,
                                 const int32_t* ranks, const float* scalings,
                                 const int32_t* token_order, const int32_t* slot_indptr,
                                 int32_t T, int32_t vocab, int32_t slots, int32_t R,
                                 const int32_t* out_slices, int32_t num_slices, int32_t regime,
                                 uint32_t* err_flags, void* stream) {
  const char* op = "lora_apply_embedding";
  lora::BgmvParams p = {};
  int out = 0;
  if (vocab <= 0) return fail(LORA_ERR_INVALID, "%s: vocab = %d must be positive", op, vocab);
  lora_status st =
      check_common(op, T, 8, slots, R, num_slices, out_slices, true, p.slice_off, &out);
  if (st != LORA_OK) return st;
  if (T == 0 || slots == 0) return ok();
  st = check_ptrs(op, {{y, "y"}, {a, "a"}, {b, "b"}},
                  {{ids, "ids"}, {ranks, "ranks"}, {scalings, "scalings"},
                   {token_order, "token_order"}, {slot_indptr, "slot_indptr"}});
  if (st != LORA_OK) return st;
  if (err_flags != nullptr && !aligned4(err_flags))
    return fail(LORA_ERR_INVALID, "%s: err_flags is not 4-byte aligned", op);
  const int reg = resolve(regime, LORA_OP_APPLY_EMBEDDING, T, slots, R, num_slices);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (reg == LORA_REGIME_STREAM) {
    if (!lora::stream_supported(R))
      return fail(LORA_ERR_UNSUPPORTED, "%s: the STREAM regime needs roundup(R, 16) <= %d", op,
                  lora::kStMaxRp);
    lora::StreamParams q = {};
    q.ids = ids; q.y = y; q.a = a; q.b = b; q.ranks = ranks; q.scalings = scalings;
    q.token_order = token_order; q.slot_indptr = slot_indptr; q.flags = err_flags;
    q.T = T; q.vocab = vocab; q.slots = slots; q.R = R; q.S = num_slices; q.out = out;
    for (int i = 0; i <= LORA_MAX_SLICES; ++i) q.slice_off[i] = p.slice_off[i];
    const char* why = nullptr;
    cudaError_t err = lora::stream_launch(q, s, true, &why);
    if (err != cudaSuccess) return cuda_fail(err, op, why);
    return ok();
  }
  if (reg == LORA_REGIME_SGMV) {
    if (!lora::sgmv_supported(num_slices, R))
      return fail(LORA_ERR_UNSUPPORTED, "%s: %s", op, lora::kSgmvShapeRule);
    const char* why = nullptr;
    cudaError_t err = lora::sgmv_expand_launch(y, nullptr, 1, ids, a, b, ranks, scalings,
                                               token_order, slot_indptr, T, vocab, slots, R,
                                               num_slices, p.slice_off, out, err_flags, s, &why);
    if (err != cudaSuccess) return cuda_fail(err, op, why);
    return ok();
  }
  if (!bgmv_fits(num_slices, R))
    return fail(LORA_ERR_UNSUPPORTED, "%s: num_slices*roundup(R,16) = %d > %d", op,
                num_slices * lora::round_up_i(R, 16), lora::kMaxSRp);
  p.ids = ids; p.y = y; p.a = a; p.b = b; p.ranks = ranks; p.scalings = scalings;
  p.token_order = token_order; p.slot_indptr = slot_indptr; p.flags = err_flags; p.T = T;
  p.in = vocab; p.slots = slots; p.R = R; p.S = num_slices; p.out = out;
  const char* why = nullptr;
  cudaError_t err = lora::bgmv_launch(lora::kModeEmbed, p, linear_items_bound(T, slots, lora::kTT),
                                      s, &why);
  if (err != cudaSuccess) return cuda_fail(err, op, why);
  return ok();
}

lora_status lora_expert_apply(const void* x_sorted, void* y_sorted, const void* a, const void* b,
                              const int32_t* pair_index, const int32_t* ranks,
                              const float* scalings, const int32_t* row_slot,
                              const int32_t* expert_offsets, int32_t rows_cap, int32_t in_features,
                              int32_t num_experts, int32_t slots, int32_t num_pairs, int32_t R,
                              const int32_t* out_slices, int32_t num_slices, void* workspace,
                              size_t workspace_bytes, uint32_t* err_flags, void* stream) {
  const char* op = "lora_expert_apply";
  lora::BgmvParams p = {};
  int out = 0;
  if (num_experts < 0 || num_experts > LORA_MAX_EXPERTS)
    return fail(num_experts < 0 ? LORA_ERR_INVALID : LORA_ERR_UNSUPPORTED,
                "%s: num_experts = %d outside [0, %d]", op, num_experts, LORA_MAX_EXPERTS);
  if (num_pairs < 0) return fail(LORA_ERR_INVALID, "%s: num_pairs = %d < 0", op, num_pairs);
  lora_status st = check_common(op, rows_cap, in_features, slots, R, num_slices, out_slices, true,
                                p.slice_off, &out);
  if (st != LORA_OK) return st;
  if (rows_cap == 0 || slots == 0 || num_experts == 0 || num_pairs == 0) return ok();
  st = check_ptrs(op, {{x_sorted, "x_sorted"}, {y_sorted, "y_sorted"}, {a, "a"}, {b, "b"}},
                  {{pair_index, "pair_index"}, {ranks, "ranks"}, {scalings, "scalings"},
                   {row_slot, "row_slot"}, {expert_offsets, "expert_offsets"}});
  if (st != LORA_OK) return st;
  if (err_flags != nullptr && !aligned4(err_flags))
    return fail(LORA_ERR_INVALID, "%s: err_flags is not 4-byte aligned", op);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const size_t gneed = expert_group_need(rows_cap, R, num_slices);
  if (workspace != nullptr && gneed > 0 && workspace_bytes >= gneed &&
      (long long)slots * num_experts <= lora::kMoeMaxGroups && in_features >= 64 &&
      lora::stream_supported(R)) {
    // grouped fold: rows sorted by (slot, expert), then the short-segment
    // (or SGMV) shrink and the streamed expand over the groups' segments
    if (!aligned16(workspace))
      return fail(LORA_ERR_INVALID, "%s: workspace is not 16-byte aligned", op);
    const int G = slots * num_experts;
    char* w = static_cast<char*>(workspace);
    int* tok = reinterpret_cast<int*>(w);
    int* seg_lo = reinterpret_cast<int*>(w + ((size_t)rows_cap * 4 + 255) / 256 * 256);
    int* seg_hi = seg_lo + lora::kMoeMaxGroups;
    int* g_rank = seg_hi + lora::kMoeMaxGroups;
    float* g_scal = reinterpret_cast<float*>(g_rank + lora::kMoeMaxGroups);
    float* hws = g_scal + lora::kMoeMaxGroups;
    cudaError_t err = lora::moe_group_launch(expert_offsets, pair_index, row_slot, ranks,
                                             scalings, rows_cap, num_experts, slots, num_pairs,
                                             R, tok, seg_lo, seg_hi, g_rank, g_scal, err_flags, s);
    if (err != cudaSuccess) return cuda_fail(err, op, nullptr);
    const lora::SgmvGroups groups = {seg_hi, pair_index, num_pairs};
    const char* why = nullptr;
    int ks = 1;
    if (lora::group_shrink_supported(num_slices, R, in_features)) {
      // the groups are short: 16-row tiles, the features split into chunks
      err = lora::group_shrink_launch(x_sorted, a, hws, tok, seg_lo, seg_hi, pair_index, g_rank,
                                      g_scal, rows_cap, in_features, G, R, num_slices, &ks, s,
                                      false);
    } else {
      // live groups are about the pairs in use: split the shrink to fill the SMs
      ks = lora::sgmv_shrink_splits(0, num_pairs < G ? num_pairs : G, in_features);
      err = lora::sgmv_shrink_launch(x_sorted, a, hws, g_rank, tok, seg_lo, rows_cap,
                                     in_features, G, R, num_slices, err_flags, s, &why, ks,
                                     g_scal, &groups);
    }
    if (err != cudaSuccess) return cuda_fail(err, op, why);
    // the expand: the groups are short (a few dozen rows), so their y rows are
    // streamed with 16-row MMA tiles rather than tiled by 128
    lora::StreamParams q = {};
    q.h = hws; q.h_split = (size_t)rows_cap * num_slices * R; q.ksplit = ks;
    q.y = y_sorted; q.b = b; q.ranks = g_rank; q.scalings = g_scal; q.token_order = tok;
    q.slot_indptr = seg_lo; q.seg_hi = seg_hi; q.slot_map = pair_index; q.flags = err_flags;
    q.T = rows_cap; q.vocab = 0; q.slots = G; q.R = R; q.S = num_slices; q.out = out;
    for (int i = 0; i <= LORA_MAX_SLICES; ++i) q.slice_off[i] = p.slice_off[i];
    err = lora::stream_launch(q, s, false, &why);
    if (err != cudaSuccess) return cuda_fail(err, op, why);
    return ok();
  }
  if (!bgmv_fits(num_slices, R))
    return fail(LORA_ERR_UNSUPPORTED, "%s: num_slices*roundup(R,16) = %d > %d", op,
                num_slices * lora::round_up_i(R, 16), lora::kMaxSRp);
  p.x = x_sorted; p.y = y_sorted; p.a = a; p.b = b; p.pair_index = pair_index; p.ranks = ranks;
  p.scalings = scalings; p.row_slot = row_slot; p.expert_offsets = expert_offsets;
  p.flags = err_flags; p.T = rows_cap; p.in = in_features; p.slots = slots; p.R = R;
  p.S = num_slices; p.out = out; p.num_experts = num_experts; p.num_pairs = num_pairs;
  const char* why = nullptr;
  // one CTA per work item (a chunk of one expert's rows)
  const int bound = linear_items_bound(rows_cap, num_experts, lora::kTT);
  cudaError_t err = lora::bgmv_launch(lora::kModeExpertSolo, p, bound, s, &why);
  if (err != cudaSuccess) return cuda_fail(err, op, why);
  return ok();
}

lora_status lora_plan_linear(const int32_t* slot_indptr, const int32_t* ranks,
                             const float* scalings, int32_t T, int32_t slots, int32_t R,
                             int32_t tile, int32_t* plan_out, int32_t plan_cap,
                             int32_t* plan_count, uint32_t* err_flags, void* stream) {
  const char* op = "lora_plan_linear";
  if (T < 0 || slots < 0 || R < 0 || tile <= 0 || plan_cap < 0)
    return fail(LORA_ERR_INVALID, "%s: negative size or tile <= 0", op);
  if (slots > LORA_MAX_SLOTS)
    return fail(LORA_ERR_UNSUPPORTED, "%s: slots = %d > %d", op, slots, LORA_MAX_SLOTS);
  lora_status st = check_ptrs(op, {}, {{slot_indptr, "slot_indptr"}, {ranks, "ranks"},
                                       {plan_count, "plan_count"}});
  if (st != LORA_OK) return st;
  if (plan_cap > 0 && plan_out == nullptr) return fail(LORA_ERR_INVALID, "%s: plan_out is NULL", op);
  cudaError_t err = lora::plan_linear_launch(slot_indptr, ranks, scalings, T, slots, R, tile,
                                             plan_out, plan_cap, plan_count, err_flags,
                                             reinterpret_cast<cudaStream_t>(stream));
  if (err != cudaSuccess) return cuda_fail(err, op, nullptr);
  return ok();
}

lora_status lora_plan_expert(const int32_t* expert_offsets, const int32_t* pair_index,
                             int32_t rows_cap, int32_t num_experts, int32_t slots,
                             int32_t max_rows, int32_t* plan_out, int32_t plan_cap,
                             int32_t* plan_count, uint32_t* err_flags, void* stream) {
  const char* op = "lora_plan_expert";
  if (rows_cap < 0 || num_experts < 0 || slots < 0 || max_rows <= 0 || plan_cap < 0)
    return fail(LORA_ERR_INVALID, "%s: negative size or max_rows <= 0", op);
  if (num_experts > LORA_MAX_EXPERTS)
    return fail(LORA_ERR_UNSUPPORTED, "%s: num_experts = %d > %d", op, num_experts,
                LORA_MAX_EXPERTS);
  lora_status st = check_ptrs(op, {}, {{expert_offsets, "expert_offsets"},
                                       {pair_index, "pair_index"}, {plan_count, "plan_count"}});
  if (st != LORA_OK) return st;
  if (plan_cap > 0 && plan_out == nullptr) return fail(LORA_ERR_INVALID, "%s: plan_out is NULL", op);
  cudaError_t err = lora::plan_expert_launch(expert_offsets, pair_index, rows_cap, num_experts,
                                             slots, max_rows, plan_out, plan_cap, plan_count,
                                             err_flags, reinterpret_cast<cudaStream_t>(stream));
  if (err != cudaSuccess) return cuda_fail(err, op, nullptr);
  return ok();
}

}  // extern "C"
