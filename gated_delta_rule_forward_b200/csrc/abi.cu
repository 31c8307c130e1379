// libgdr C ABI: argument validation, kernel selection, launch-error mapping.
// The operation each entry point performs is specified in include/gdr.h.
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <string>

#include "common.cuh"
#include "gdr.h"
#include "chunk_bwd.cuh"
#include "chunk_split.cuh"

namespace {

thread_local std::string g_last_error;

gdr_status_t fail(gdr_status_t st, const std::string &why) {
  g_last_error = why;
  return st;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool injected_launch_fault() {
  const char *f = std::getenv("GDR_FAULT");
  return f && std::strcmp(f, "launch") == 0;
}

gdr_status_t check_cuda(cudaError_t e, const char *what) {
  if (e == cudaSuccess) return GDR_OK;
  return fail(GDR_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

bool valid_variant(int v) { return v >= GDR_DELTANET && v <= GDR_KLA; }

// The raw-input flag may be OR'ed into a variant: returns it and strips it.
bool take_raw(int &variant) {
  const bool raw = (variant & GDR_RAW_INPUTS) != 0;
  variant &= ~GDR_RAW_INPUTS;
  return raw;
}
bool valid_dim(int d) { return d == 64 || d == 128; }

enum class Kernel { None, Token, Split };

bool split_ok(int variant, int dtype, int dk, int dv) {
  return dtype == GDR_BF16 && gdr_split_supported(variant, dk, dv);
}

// Which kernel a forward call runs, or None with a status and reason.  `ws`
// is the workspace the caller passes; the automatic choice takes the
// chunked path only when the workspace is large enough for it.
Kernel select_forward(int variant, int dtype, int B, int T, int H, int dk, int dv, int chunk, size_t ws,
                      gdr_status_t *st, std::string *why) {
  *st = GDR_OK;
  const bool sp = split_ok(variant, dtype, dk, dv);
  const size_t need = sp ? gdr_split_workspace_bytes(variant, B, T, H, dv) : 0;
  if (chunk == 1) return Kernel::Token;
  if (chunk == 0) return (sp && ws >= need) ? Kernel::Split : Kernel::Token;
  if (chunk == 65) {
    if (!sp) {
      *st = GDR_ERR_UNSUPPORTED;
      *why = "chunk=65 (the chunked path) needs bf16 I/O and dk = 128";
      return Kernel::None;
    }
    if (ws < need) {
      *st = GDR_ERR_INVALID_ARG;
      *why = "chunk=65 needs gdr_forward_workspace_size() bytes of workspace";
      return Kernel::None;
    }
    return Kernel::Split;
  }
  if (chunk == 64) {
    *st = GDR_ERR_UNSUPPORTED;
    *why = "chunk=64 (a one-kernel chunked path without workspace) is not built; use 0 (auto) or 65";
    return Kernel::None;
  }
  *st = GDR_ERR_INVALID_ARG;
  *why = "chunk must be 0 (auto), 1 (per-token) or 65 (chunked)";
  return Kernel::None;
}

gdr_status_t validate_common(int variant, int dtype, int dk, int dv) {
  if (!valid_variant(variant)) return fail(GDR_ERR_INVALID_ARG, "variant out of range");
  if (dtype != GDR_F32 && dtype != GDR_BF16) return fail(GDR_ERR_INVALID_ARG, "dtype must be GDR_F32 or GDR_BF16");
  if (!valid_dim(dk) || !valid_dim(dv)) return fail(GDR_ERR_UNSUPPORTED, "dk and dv must each be 64 or 128");
  return GDR_OK;
}

gdr_status_t validate_gates(int variant, const float *beta, const float *log_g, const float *erase_b,
                            const float *write_w) {
  if (variant != GDR_GDN2 && !beta) return fail(GDR_ERR_INVALID_ARG, "beta (eta for KLA) is required");
  if (variant != GDR_DELTANET && !log_g) return fail(GDR_ERR_INVALID_ARG, "log_g is required for this variant");
  if (variant == GDR_GDN2 && (!erase_b || !write_w))
    return fail(GDR_ERR_INVALID_ARG, "GDN-2 needs erase_b and write_w");
  const void *ptrs[4] = {beta, log_g, erase_b, write_w};
  for (const void *p : ptrs)
    if (p && !aligned16(p)) return fail(GDR_ERR_ALIGNMENT, "a gate pointer is not 16-byte aligned");
  return GDR_OK;
}

}  // namespace

extern "C" {

int gdr_version(void) { return 101; }

const char *gdr_status_string(gdr_status_t s) {
  switch (s) {
    case GDR_OK: return "GDR_OK";
    case GDR_ERR_INVALID_ARG: return "GDR_ERR_INVALID_ARG";
    case GDR_ERR_UNSUPPORTED: return "GDR_ERR_UNSUPPORTED";
    case GDR_ERR_ALIGNMENT: return "GDR_ERR_ALIGNMENT";
    case GDR_ERR_CUDA: return "GDR_ERR_CUDA";
    case GDR_ERR_TIMEOUT: return "GDR_ERR_TIMEOUT";
    case GDR_ERR_RANGE: return "GDR_ERR_RANGE";
  }
  return "GDR_UNKNOWN_STATUS";
}

const char *gdr_last_error(void) { return g_last_error.c_str(); }

gdr_status_t gdr_device_status(void *stream) {
  const int ef = gdr_read_device_error(static_cast<cudaStream_t>(stream));
  const int eb = gdr_bwd_read_device_error(static_cast<cudaStream_t>(stream));
  if (ef < 0 || eb < 0) return fail(GDR_ERR_CUDA, "synchronisation or symbol read failed");
  const int e = ef | eb;
  if (e & 1) return fail(GDR_ERR_TIMEOUT, "a bounded device-side wait gave up");
  if (e & 2) return fail(GDR_ERR_RANGE, "a chunked-kernel operand left its representable range");
  return GDR_OK;
}

size_t gdr_forward_workspace_size(int variant, int dtype, int B, int T, int H, int dk, int dv, int chunk) {
  take_raw(variant);
  if (!valid_variant(variant) || !valid_dim(dk) || !valid_dim(dv) || B <= 0 || T <= 0 || H <= 0) return 0;
  if ((chunk == 0 || chunk == 65) && split_ok(variant, dtype, dk, dv)) return gdr_split_workspace_bytes(variant, B, T, H, dv);
  return 0;
}

// The kernel a call with a workspace of gdr_forward_workspace_size() bytes runs.
static Kernel planned_kernel(int variant, int dtype, int B, int T, int H, int dk, int dv, int chunk) {
  take_raw(variant);
  gdr_status_t st;
  std::string why;
  const size_t ws = gdr_forward_workspace_size(variant, dtype, B, T, H, dk, dv, chunk);
  return select_forward(variant, dtype, B, T, H, dk, dv, chunk, ws, &st, &why);
}

int gdr_forward_launches(int variant, int dtype, int B, int T, int H, int dk, int dv, int chunk) {
  take_raw(variant);
  if (!valid_variant(variant) || (dtype != 0 && dtype != 1) || !valid_dim(dk) || !valid_dim(dv)) return 0;
  if (B < 0 || T < 0 || H < 0) return 0;
  const Kernel kern = planned_kernel(variant, dtype, B, T, H, dk, dv, chunk);
  if (kern == Kernel::None) return 0;
  if ((long)B * H == 0) return 0;
  if (T == 0) return 1;  // state copy or clear
  if (kern == Kernel::Split) return gdr_split_launches(variant, B, T, H, dv);
  return 1;
}

const char *gdr_forward_kernel_name(int variant, int dtype, int B, int T, int H, int dk, int dv, int chunk) {
  if (gdr_forward_launches(variant, dtype, B, T, H, dk, dv, chunk) == 0 && (long)B * H * T != 0) return "none";
  const Kernel kern = planned_kernel(variant, dtype, B, T, H, dk, dv, chunk);
  if (kern == Kernel::Split) return "chunk64_split";
  if (kern == Kernel::Token) return dtype == GDR_BF16 ? "token_bf16io" : "token_f32io";
  return "none";
}

gdr_status_t gdr_forward_plan(int variant, int B, int T, int H, int dv, int sms, int *segments,
                              int *segment_chunks, int *split_chunk) {
  take_raw(variant);
  if (!valid_variant(variant)) return fail(GDR_ERR_INVALID_ARG, "unknown variant");
  if (!valid_dim(dv)) return fail(GDR_ERR_INVALID_ARG, "dv must be 64 or 128");
  if (B < 0 || T < 0 || H < 0 || sms < 0) return fail(GDR_ERR_INVALID_ARG, "B, T, H and sms must be >= 0");
  if (!segments || !segment_chunks || !split_chunk) return fail(GDR_ERR_INVALID_ARG, "output pointer is NULL");
  gdr_split_plan(variant, B, T, H, dv, sms, segments, segment_chunks, split_chunk);
  return GDR_OK;
}

gdr_status_t gdr_forward_segment_parts(int variant, int B, int T, int H, int dv, int sms, int *parts,
                                       int *part_chunks) {
  take_raw(variant);
  if (!valid_variant(variant)) return fail(GDR_ERR_INVALID_ARG, "unknown variant");
  if (!valid_dim(dv)) return fail(GDR_ERR_INVALID_ARG, "dv must be 64 or 128");
  if (B < 0 || T < 0 || H < 0 || sms < 0) return fail(GDR_ERR_INVALID_ARG, "B, T, H and sms must be >= 0");
  if (!parts || !part_chunks) return fail(GDR_ERR_INVALID_ARG, "output pointer is NULL");
  int g = 0, l = 0, c = 0;
  gdr_split_plan(variant, B, T, H, dv, sms, &g, &l, &c, parts, part_chunks);
  return GDR_OK;
}

gdr_status_t gdr_forward_chunked(int variant, int dtype, int B, int T, int H, int dk, int dv,
                                 const gdr_fwd_args_t *a, float eps, float scale, int chunk,
                                 void *workspace, size_t workspace_bytes, void *stream) {
  const bool raw = take_raw(variant);
  gdr_status_t st = validate_common(variant, dtype, dk, dv);
  if (st != GDR_OK) return st;
  if (B < 0 || T < 0 || H < 0) return fail(GDR_ERR_INVALID_ARG, "B, T and H must be >= 0");
  if (!a) return fail(GDR_ERR_INVALID_ARG, "args is NULL");
  if (!workspace) workspace_bytes = 0;
  if (workspace && !aligned16(workspace)) return fail(GDR_ERR_ALIGNMENT, "workspace must be 16-byte aligned");
  std::string why;
  const Kernel kern = select_forward(variant, dtype, B, T, H, dk, dv, chunk, workspace_bytes, &st, &why);
  if (kern == Kernel::None) return fail(st, why);
  if ((long)B * H == 0) return GDR_OK;  // nothing to do
  if (T > 0) {
    if (!a->q || !a->k || !a->v || !a->o) return fail(GDR_ERR_INVALID_ARG, "q, k, v and o are required");
    const void *io[4] = {a->q, a->k, a->v, a->o};
    for (const void *p : io)
      if (!aligned16(p)) return fail(GDR_ERR_ALIGNMENT, "q, k, v and o must be 16-byte aligned");
    st = validate_gates(variant, a->beta, a->log_g, a->erase_b, a->write_w);
    if (st != GDR_OK) return st;
  }
  if ((a->initial_state && !aligned16(a->initial_state)) || (a->final_state && !aligned16(a->final_state)))
    return fail(GDR_ERR_ALIGNMENT, "state pointers must be 16-byte aligned");
  if (!(eps >= 0.f)) return fail(GDR_ERR_INVALID_ARG, "eps must be >= 0");
  if (injected_launch_fault()) return fail(GDR_ERR_CUDA, "injected launch failure (GDR_FAULT=launch)");

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (T == 0) {
    // No tokens: the final state is the initial state.
    if (!a->final_state) return GDR_OK;
    const size_t bytes = (size_t)B * H * dk * dv * sizeof(float);
    if (a->initial_state == a->final_state) return GDR_OK;
    if (a->initial_state)
      return check_cuda(cudaMemcpyAsync(a->final_state, a->initial_state, bytes, cudaMemcpyDeviceToDevice, s),
                        "state copy");
    return check_cuda(cudaMemsetAsync(a->final_state, 0, bytes, s), "state clear");
  }

  gdr::FwdProblem p;
  p.variant = variant; p.B = B; p.T = T; p.H = H; p.dk = dk; p.dv = dv;
  p.bf16_io = dtype == GDR_BF16;
  p.raw = raw;
  p.q = a->q; p.k = a->k; p.v = a->v;
  p.beta = a->beta; p.log_g = a->log_g; p.erase_b = a->erase_b; p.write_w = a->write_w;
  p.s0 = a->initial_state; p.s_final = a->final_state; p.o = a->o;
  p.eps = eps; p.scale = scale;
  if (kern == Kernel::Split) {
    std::string err;
    const cudaError_t e = gdr_launch_split(p, workspace, workspace_bytes, s, &err);
    if (e != cudaSuccess) return fail(GDR_ERR_CUDA, "chunk64_split: " + err + cudaGetErrorString(e));
    return GDR_OK;
  }
  return check_cuda(gdr_launch_token_forward(p, s), "token_fwd launch");
}

gdr_status_t gdr_forward_chunked_noalloc(int variant, int dtype, int B, int T, int H, int dk, int dv,
                                         const gdr_fwd_args_t *a, float eps, float scale, void *stream) {
  const int variant_arg = variant;
  const bool raw = take_raw(variant);
  gdr_status_t st = validate_common(variant, dtype, dk, dv);
  if (st != GDR_OK) return st;
  if (B < 0 || T < 0 || H < 0) return fail(GDR_ERR_INVALID_ARG, "B, T and H must be >= 0");
  if (!a) return fail(GDR_ERR_INVALID_ARG, "args is NULL");
  if (!split_ok(variant, dtype, dk, dv))
    return fail(GDR_ERR_UNSUPPORTED,
                "the no-allocation entry point needs bf16 I/O, dk = 128 and dv in {64, 128} (all five variants)");
  // The records must fit; the segmented carry's maps are optional (without
  // room for them the call runs the unsegmented sweep).
  const size_t rec = gdr_split_record_bytes(variant, dv);
  const size_t records = (size_t)B * H * (((size_t)T + 63) / 64);
  const size_t have = gdr_split_fixed_scratch_bytes();
  if (records * rec > have)
    return fail(GDR_ERR_UNSUPPORTED,
                "problem needs " + std::to_string(records) + " records of " + std::to_string(rec) + " bytes (" +
                    std::to_string(records * rec) + " bytes) but the fixed scratch holds " + std::to_string(have) +
                    " bytes: B * H * ceil(T / 64) must be at most " + std::to_string(have / rec) +
                    " for this variant and dv");
  if ((long)B * H == 0 || T == 0) return gdr_forward_chunked(variant_arg, dtype, B, T, H, dk, dv, a, eps, scale, 65,
                                                             nullptr, 0, stream);
  if (!a->q || !a->k || !a->v || !a->o) return fail(GDR_ERR_INVALID_ARG, "q, k, v and o are required");
  const void *io[4] = {a->q, a->k, a->v, a->o};
  for (const void *p : io)
    if (!aligned16(p)) return fail(GDR_ERR_ALIGNMENT, "q, k, v and o must be 16-byte aligned");
  st = validate_gates(variant, a->beta, a->log_g, a->erase_b, a->write_w);
  if (st != GDR_OK) return st;
  if ((a->initial_state && !aligned16(a->initial_state)) || (a->final_state && !aligned16(a->final_state)))
    return fail(GDR_ERR_ALIGNMENT, "state pointers must be 16-byte aligned");
  if (!(eps >= 0.f)) return fail(GDR_ERR_INVALID_ARG, "eps must be >= 0");
  if (injected_launch_fault()) return fail(GDR_ERR_CUDA, "injected launch failure (GDR_FAULT=launch)");
  void *scratch = nullptr;
  cudaError_t e = gdr_split_fixed_scratch(&scratch);
  if (e != cudaSuccess) return fail(GDR_ERR_CUDA, std::string("fixed scratch lookup: ") + cudaGetErrorString(e));
  gdr::FwdProblem p;
  p.variant = variant; p.B = B; p.T = T; p.H = H; p.dk = dk; p.dv = dv;
  p.bf16_io = true;
  p.raw = raw;
  p.q = a->q; p.k = a->k; p.v = a->v;
  p.beta = a->beta; p.log_g = a->log_g; p.erase_b = a->erase_b; p.write_w = a->write_w;
  p.s0 = a->initial_state; p.s_final = a->final_state; p.o = a->o;
  p.eps = eps; p.scale = scale;
  std::string err;
  e = gdr_launch_split(p, scratch, have, static_cast<cudaStream_t>(stream), &err);
  if (e != cudaSuccess) return fail(GDR_ERR_CUDA, "chunk64_split: " + err + cudaGetErrorString(e));
  return GDR_OK;
}

size_t gdr_backward_workspace_size(int variant, int dtype, int B, int T, int H, int dk, int dv) {
  if (variant & GDR_RAW_INPUTS) return 0;
  if (!gdr_bwd_supported(variant, dtype == GDR_BF16, dk, dv) || B <= 0 || T <= 0 || H <= 0) return 0;
  return gdr_bwd_workspace_bytes(variant, B, T, H, dv);
}

gdr_status_t gdr_backward(int variant, int dtype, int B, int T, int H, int dk, int dv, const gdr_fwd_args_t *a,
                          const void *d_o, const float *d_final, const gdr_bwd_grads_t *g, float eps, float scale,
                          void *workspace, size_t workspace_bytes, void *stream) {
  if (variant & GDR_RAW_INPUTS) return fail(GDR_ERR_UNSUPPORTED, "the backward takes transformed inputs (no GDR_RAW_INPUTS)");
  gdr_status_t st = validate_common(variant, dtype, dk, dv);
  if (st != GDR_OK) return st;
  if (!gdr_bwd_supported(variant, dtype == GDR_BF16, dk, dv))
    return fail(GDR_ERR_UNSUPPORTED,
                "the backward needs bf16 I/O, dk = 128 and dv in {64, 128}");
  if (B < 0 || T < 0 || H < 0) return fail(GDR_ERR_INVALID_ARG, "B, T and H must be >= 0");
  if (!a || !g) return fail(GDR_ERR_INVALID_ARG, "args and grads are required");
  if ((long)B * H == 0) return GDR_OK;
  if ((a->initial_state && !aligned16(a->initial_state)) || (d_final && !aligned16(d_final)) ||
      (g->d_initial_state && !aligned16(g->d_initial_state)))
    return fail(GDR_ERR_ALIGNMENT, "state pointers must be 16-byte aligned");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (T == 0) {   // no tokens: the initial state's gradient is the final state's
    if (!g->d_initial_state) return GDR_OK;
    const size_t bytes = (size_t)B * H * dk * dv * sizeof(float);
    if (d_final)
      return check_cuda(cudaMemcpyAsync(g->d_initial_state, d_final, bytes, cudaMemcpyDeviceToDevice, s),
                        "state gradient copy");
    return check_cuda(cudaMemsetAsync(g->d_initial_state, 0, bytes, s), "state gradient clear");
  }
  if (!a->q || !a->k || !a->v || !d_o || !g->dq || !g->dk || !g->dv)
    return fail(GDR_ERR_INVALID_ARG, "q, k, v, d_o, dq, dk and dv are required");
  if (variant != GDR_GDN2 && !g->dbeta) return fail(GDR_ERR_INVALID_ARG, "dbeta is required for this variant");
  if (variant == GDR_GDN2 && (!g->d_erase_b || !g->d_write_w))
    return fail(GDR_ERR_INVALID_ARG, "GDN-2 needs d_erase_b and d_write_w");
  if (variant != GDR_DELTANET && !g->dlog_g) return fail(GDR_ERR_INVALID_ARG, "dlog_g is required for this variant");
  const void *ptrs[11] = {a->q, a->k, a->v, d_o, g->dq, g->dk, g->dv, g->dbeta, g->dlog_g, g->d_erase_b,
                          g->d_write_w};
  for (const void *p : ptrs)
    if (p && !aligned16(p)) return fail(GDR_ERR_ALIGNMENT, "tensor pointers must be 16-byte aligned");
  st = validate_gates(variant, a->beta, a->log_g, a->erase_b, a->write_w);
  if (st != GDR_OK) return st;
  if (!(eps >= 0.f)) return fail(GDR_ERR_INVALID_ARG, "eps must be >= 0");
  if (!workspace || !aligned16(workspace)) return fail(GDR_ERR_INVALID_ARG, "a 16-byte aligned workspace is required");
  if (workspace_bytes < gdr_bwd_workspace_bytes(variant, B, T, H, dv))
    return fail(GDR_ERR_INVALID_ARG, "the workspace must be at least gdr_backward_workspace_size() bytes");
  if (injected_launch_fault()) return fail(GDR_ERR_CUDA, "injected launch failure (GDR_FAULT=launch)");
  gdr::BwdProblem p;
  p.f.variant = variant; p.f.B = B; p.f.T = T; p.f.H = H; p.f.dk = dk; p.f.dv = dv;
  p.f.bf16_io = true;
  p.f.raw = false;
  p.f.q = a->q; p.f.k = a->k; p.f.v = a->v;
  p.f.beta = a->beta; p.f.log_g = a->log_g;
  p.f.erase_b = variant == GDR_GDN2 ? a->erase_b : nullptr;
  p.f.write_w = variant == GDR_GDN2 ? a->write_w : nullptr;
  p.f.s0 = a->initial_state; p.f.s_final = nullptr; p.f.o = nullptr;
  p.f.eps = eps; p.f.scale = scale;
  p.d_o = d_o; p.d_final = d_final;
  p.dq = g->dq; p.dk = g->dk; p.dv = g->dv;
  p.dbeta = g->dbeta; p.dlog_g = variant == GDR_DELTANET ? nullptr : g->dlog_g;
  p.d_s0 = g->d_initial_state;
  p.d_erase = variant == GDR_GDN2 ? g->d_erase_b : nullptr;
  p.d_write = variant == GDR_GDN2 ? g->d_write_w : nullptr;
  std::string err;
  const cudaError_t e = gdr_launch_backward(p, workspace, workspace_bytes, s, &err);
  if (e != cudaSuccess) return fail(GDR_ERR_CUDA, "backward: " + err + cudaGetErrorString(e));
  return GDR_OK;
}

gdr_status_t gdr_decode_step(int variant, int dtype, int N, int H, int dk, int dv, const void *q, const void *k,
                             const void *v, const float *beta, const float *log_g, const float *erase_b,
                             const float *write_w, float *state, void *o, float eps, float scale, void *stream) {
  const bool raw = take_raw(variant);
  gdr_status_t st = validate_common(variant, dtype, dk, dv);
  if (st != GDR_OK) return st;
  if (N < 0 || H < 0) return fail(GDR_ERR_INVALID_ARG, "N and H must be >= 0");
  if ((long)N * H == 0) return GDR_OK;
  if (!q || !k || !v || !o || !state) return fail(GDR_ERR_INVALID_ARG, "q, k, v, o and state are required");
  const void *io[5] = {q, k, v, o, state};
  for (const void *p : io)
    if (!aligned16(p)) return fail(GDR_ERR_ALIGNMENT, "q, k, v, o and state must be 16-byte aligned");
  st = validate_gates(variant, beta, log_g, erase_b, write_w);
  if (st != GDR_OK) return st;
  if (!(eps >= 0.f)) return fail(GDR_ERR_INVALID_ARG, "eps must be >= 0");
  if (injected_launch_fault()) return fail(GDR_ERR_CUDA, "injected launch failure (GDR_FAULT=launch)");
  gdr::DecodeProblem p;
  p.variant = variant; p.N = N; p.H = H; p.dk = dk; p.dv = dv;
  p.bf16_io = dtype == GDR_BF16;
  p.raw = raw;
  p.q = q; p.k = k; p.v = v;
  p.beta = beta; p.log_g = log_g; p.erase_b = erase_b; p.write_w = write_w;
  p.state = state; p.o = o; p.eps = eps; p.scale = scale;
  return check_cuda(gdr_launch_decode(p, static_cast<cudaStream_t>(stream)), "decode launch");
}

}  // extern "C"
