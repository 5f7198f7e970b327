// gdr2_api.cu -- the extern "C" entry points of libgdr2.so.
//
// Host-side argument validation, the per-device status word and the
// dispatch to the kernels. Nothing here allocates device memory.

#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <atomic>
#include <mutex>

#include "../../include/gdr2.h"
#include "gdr2_common.cuh"
#include "gdr2_launch.h"

namespace {

thread_local char g_last_error[512] = "";

gdr2_status fail(gdr2_status st, const char *fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
    va_end(ap);
    return st;
}

// One status word per device. Kernels OR bits into it (gdr2::kStatus*).
__device__ unsigned g_status_word;

constexpr int kMaxDevices = 64;
unsigned *g_status_ptr[kMaxDevices];

std::mutex g_status_mu;

// The status word's device address on `dev` (current). Only a successful lookup is kept.
unsigned *status_ptr(int dev)
{
    if (dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_status_mu);
    if (!g_status_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_status_word) == cudaSuccess) g_status_ptr[dev] = static_cast<unsigned *>(p);
    }
    return g_status_ptr[dev];
}

std::atomic<int> g_debug_giveup{0};
std::atomic<int> g_debug_unfused{0};

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

gdr2_status check_dims(int B, int T, int H, int dk, int dv)
{
    if (B < 0 || T < 0 || H < 0) return fail(GDR2_ERR_INVALID_ARG, "negative size (B=%d T=%d H=%d)", B, T, H);
    if (dk <= 0 || dv <= 0) return fail(GDR2_ERR_INVALID_ARG, "dk and dv must be positive (dk=%d dv=%d)", dk, dv);
    if ((dk != 64 && dk != 128) || (dv != 64 && dv != 128))
        return fail(GDR2_ERR_UNSUPPORTED, "dk and dv must be 64 or 128 (dk=%d dv=%d)", dk, dv);
    if ((long long)B * T * H * (dk > dv ? dk : dv) > (1ll << 40))
        return fail(GDR2_ERR_INVALID_ARG, "problem too large");
    return GDR2_OK;
}

gdr2_status check_ptr(const void *p, const char *name, bool nullable)
{
    if (!p) return nullable ? GDR2_OK : fail(GDR2_ERR_INVALID_ARG, "%s is NULL", name);
    if (!aligned16(p)) return fail(GDR2_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);
    return GDR2_OK;
}

gdr2_status check_gates(int gates)
{
    if (gates < 0 || gates > (GDR2_GATE_SCALAR_B | GDR2_GATE_SCALAR_W))
        return fail(GDR2_ERR_INVALID_ARG, "gates must combine GDR2_GATE_SCALAR_B and GDR2_GATE_SCALAR_W (got %d)",
                    gates);
    return GDR2_OK;
}

// A vector gate is read by tiles (16-byte aligned, like every tensor); a scalar gate
// ([..., T, H], one value per token-head) element by element.
gdr2_status check_gate_ptr(const void *p, const char *name, bool nullable, int scalar, gdr2_dtype dt)
{
    if (!scalar) return check_ptr(p, name, nullable);
    if (!p && !nullable) return fail(GDR2_ERR_INVALID_ARG, "%s is NULL", name);
    const uintptr_t esz = dt == GDR2_BF16 ? 2 : 4;
    if ((reinterpret_cast<uintptr_t>(p) & (esz - 1)) != 0)
        return fail(GDR2_ERR_INVALID_ARG, "%s is not aligned to its element size", name);
    return GDR2_OK;
}

#define GDR2_TRY(expr)                      \
    do {                                    \
        gdr2_status st_ = (expr);           \
        if (st_ != GDR2_OK) return st_;     \
    } while (0)

gdr2_status check_dtype(gdr2_dtype dt)
{
    if (dt != GDR2_F32 && dt != GDR2_BF16) return fail(GDR2_ERR_INVALID_ARG, "unknown dtype %d", (int)dt);
    return GDR2_OK;
}

gdr2_status device_status(unsigned **out)
{
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(GDR2_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    *out = status_ptr(dev);
    if (!*out) return fail(GDR2_ERR_CUDA, "cannot resolve the device status word on device %d", dev);
    return GDR2_OK;
}

gdr2_status launched(cudaError_t e, const char *what)
{
    if (e != cudaSuccess) return fail(GDR2_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
    g_last_error[0] = '\0';
    return GDR2_OK;
}

}  // namespace

namespace gdr2 {
int debug_giveup_flag() { return g_debug_giveup.load(); }
int debug_unfused_flag() { return g_debug_unfused.load(); }
}  // namespace gdr2

extern "C" {

int gdr2_abi_version(void) { return GDR2_ABI_VERSION; }

void gdr2_debug_force_timeout(int enable) { g_debug_giveup.store(enable != 0 ? 1 : 0); }

void gdr2_debug_forward_unfused(int enable) { g_debug_unfused.store(enable != 0 ? 1 : 0); }

gdr2_status gdr2_debug_recip(const float *x, float *y, long long n, void *stream)
{
    if (n < 0) return fail(GDR2_ERR_INVALID_ARG, "n must not be negative (n=%lld)", n);
    if (n == 0) return GDR2_OK;
    if (!x || !y) return fail(GDR2_ERR_INVALID_ARG, "x and y must not be NULL");
    return launched(gdr2::launch_recip_eval(x, y, n, static_cast<cudaStream_t>(stream)), "gdr2_debug_recip");
}

const char *gdr2_last_error(void) { return g_last_error; }

size_t gdr2_forward_workspace_bytes(int B, int T, int H, int dk, int dv, gdr2_dtype dt)
{
    if (B < 0 || T < 0 || H < 0) return 0;
    if (dt != GDR2_BF16 || dk != 128 || dv != 128) return 0;
    return gdr2::forward_tc_workspace_bytes(B, T, H);
}

// All forward entry points: dense (cu_seqlens = NULL) or packed, gates, epilogue.
static gdr2_status forward_impl(const char *who, int B, int T, int H, int dk, int dv, gdr2_dtype dt, int gates,
                                const int *cu_seqlens, bool packed, const void *q, const void *k, const void *v,
                                const float *log_alpha, const void *b, const void *w, const float *S0,
                                const void *out_gate, const float *norm_weight, float norm_eps, void *o, float *S_T,
                                float *saved_states, void *workspace, size_t workspace_bytes, void *stream)
{
    GDR2_TRY(check_dims(B, T, H, dk, dv));
    GDR2_TRY(check_dtype(dt));
    GDR2_TRY(check_gates(gates));
    const bool epilogue = out_gate || norm_weight;
    const bool tc_shape = dt == GDR2_BF16 && dk == 128 && dv == 128;
    if (packed && !tc_shape)
        return fail(GDR2_ERR_UNSUPPORTED, "%s: packed sequences need bf16 inputs with dk = dv = 128", who);
    if (epilogue && !tc_shape)
        return fail(GDR2_ERR_UNSUPPORTED, "%s: the output norm and gate need bf16 inputs with dk = dv = 128", who);
    if ((long long)B * H == 0) return GDR2_OK;
    const bool has_tokens = (long long)B * T * H > 0;
    if (packed) {
        if (!cu_seqlens) return fail(GDR2_ERR_INVALID_ARG, "cu_seqlens is NULL");
        if ((reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) != 0)
            return fail(GDR2_ERR_INVALID_ARG, "cu_seqlens is not 4-byte aligned");
    }
    GDR2_TRY(check_ptr(q, "q", !has_tokens));
    GDR2_TRY(check_ptr(k, "k", !has_tokens));
    GDR2_TRY(check_ptr(v, "v", !has_tokens));
    GDR2_TRY(check_ptr(log_alpha, "log_alpha", !has_tokens));
    GDR2_TRY(check_gate_ptr(b, "b", !has_tokens, gates & GDR2_GATE_SCALAR_B, dt));
    GDR2_TRY(check_gate_ptr(w, "w", !has_tokens, gates & GDR2_GATE_SCALAR_W, dt));
    GDR2_TRY(check_ptr(o, "o", !has_tokens));
    GDR2_TRY(check_ptr(S0, "S0", true));
    GDR2_TRY(check_ptr(S_T, "S_T", true));
    GDR2_TRY(check_ptr(saved_states, "saved_states", true));
    GDR2_TRY(check_ptr(out_gate, "out_gate", true));
    if (norm_weight) {
        if ((reinterpret_cast<uintptr_t>(norm_weight) & 3u) != 0)
            return fail(GDR2_ERR_INVALID_ARG, "norm_weight is not 4-byte aligned");
        if (!(norm_eps >= 0.f && norm_eps <= 3.4e38f))
            return fail(GDR2_ERR_INVALID_ARG, "norm_eps must be finite and >= 0 (got %g)", (double)norm_eps);
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (T == 0) {
        // No tokens: S_T = S0 (or zeros); nothing to save.
        if (S_T && S_T != S0) {
            const size_t bytes = (size_t)B * H * dk * dv * sizeof(float);
            cudaError_t e = S0 ? cudaMemcpyAsync(S_T, S0, bytes, cudaMemcpyDeviceToDevice, s)
                               : cudaMemsetAsync(S_T, 0, bytes, s);
            return launched(e, who);
        }
        return GDR2_OK;
    }
    const size_t need = packed ? gdr2_forward_varlen_workspace_bytes(B, T, H, dk, dv, dt)
                               : gdr2_forward_workspace_bytes(B, T, H, dk, dv, dt);
    if (need > 0) {
        if (!workspace || workspace_bytes < need)
            return fail(GDR2_ERR_INVALID_ARG, "workspace too small: %zu bytes given, %zu needed", workspace_bytes,
                        need);
        if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
            return fail(GDR2_ERR_INVALID_ARG, "workspace is not 256-byte aligned");
    }
    gdr2::FwdArgs a{B,         T,         H,       dk,       dv,     dt == GDR2_BF16,
                    q,         k,         v,       log_alpha, b,     w,
                    S0,        o,         S_T,     saved_states, workspace, workspace_bytes,
                    nullptr,   packed ? cu_seqlens : nullptr, gates, out_gate, norm_weight, norm_eps};
    GDR2_TRY(device_status(&a.status));
    if (gdr2::forward_tc_supported(a)) return launched(gdr2::launch_forward_tc(a, s), who);
    if (packed || epilogue)
        return fail(GDR2_ERR_UNSUPPORTED, "%s: the tensor-core forward is not available on this device", who);
    return launched(gdr2::launch_forward_simt(a, s), who);
}

gdr2_status gdr2_forward_gated(int B, int T, int H, int dk, int dv, gdr2_dtype dt, int gates, const void *q,
                               const void *k, const void *v, const float *log_alpha, const void *b, const void *w,
                               const float *S0, void *o, float *S_T, float *saved_states, void *workspace,
                               size_t workspace_bytes, void *stream)
{
    return forward_impl("gdr2_forward", B, T, H, dk, dv, dt, gates, nullptr, false, q, k, v, log_alpha, b, w, S0,
                        nullptr, nullptr, 0.f, o, S_T, saved_states, workspace, workspace_bytes, stream);
}

gdr2_status gdr2_forward(int B, int T, int H, int dk, int dv, gdr2_dtype dt, const void *q, const void *k,
                         const void *v, const float *log_alpha, const void *b, const void *w, const float *S0,
                         void *o, float *S_T, float *saved_states, void *workspace, size_t workspace_bytes,
                         void *stream)
{
    return gdr2_forward_gated(B, T, H, dk, dv, dt, 0, q, k, v, log_alpha, b, w, S0, o, S_T, saved_states,
                              workspace, workspace_bytes, stream);
}

size_t gdr2_forward_varlen_workspace_bytes(int N, int T, int H, int dk, int dv, gdr2_dtype dt)
{
    if (N < 0 || T < 0 || H < 0) return 0;
    if (dt != GDR2_BF16 || dk != 128 || dv != 128) return 0;
    return gdr2::forward_tc_varlen_workspace_bytes(N, T, H);
}

gdr2_status gdr2_forward_varlen(int N, int T, int H, int dk, int dv, gdr2_dtype dt, int gates, const int *cu_seqlens,
                                const void *q, const void *k, const void *v, const float *log_alpha, const void *b,
                                const void *w, const float *S0, void *o, float *S_T, float *saved_states,
                                void *workspace, size_t workspace_bytes, void *stream)
{
    return forward_impl("gdr2_forward_varlen", N, T, H, dk, dv, dt, gates, cu_seqlens, true, q, k, v, log_alpha, b,
                        w, S0, nullptr, nullptr, 0.f, o, S_T, saved_states, workspace, workspace_bytes, stream);
}

gdr2_status gdr2_forward_ex(int B, int T, int H, int dk, int dv, gdr2_dtype dt, int gates, const int *cu_seqlens,
                            const void *q, const void *k, const void *v, const float *log_alpha, const void *b,
                            const void *w, const float *S0, const void *out_gate, const float *norm_weight,
                            float norm_eps, void *o, float *S_T, float *saved_states, void *workspace,
                            size_t workspace_bytes, void *stream)
{
    return forward_impl("gdr2_forward_ex", B, T, H, dk, dv, dt, gates, cu_seqlens, cu_seqlens != nullptr, q, k, v,
                        log_alpha, b, w, S0, out_gate, norm_weight, norm_eps, o, S_T, saved_states, workspace,
                        workspace_bytes, stream);
}

gdr2_status gdr2_short_conv_silu(int N, int T, int H, int d, gdr2_dtype dt, int width, int l2norm, float l2_eps,
                                 const int *cu_seqlens, const void *x, const float *weight, const void *state_in,
                                 void *state_out, void *y, void *stream)
{
    GDR2_TRY(check_dtype(dt));
    if (N < 0 || T < 0 || H < 0) return fail(GDR2_ERR_INVALID_ARG, "negative size (N=%d T=%d H=%d)", N, T, H);
    if (d != 64 && d != 128) return fail(GDR2_ERR_UNSUPPORTED, "d must be 64 or 128 (d=%d)", d);
    if (width < 1 || width > 4) return fail(GDR2_ERR_UNSUPPORTED, "width must be 1 .. 4 (width=%d)", width);
    if (l2norm != 0 && l2norm != 1) return fail(GDR2_ERR_INVALID_ARG, "l2norm must be 0 or 1");
    if (!(l2_eps >= 0.f && l2_eps <= 3.4e38f))
        return fail(GDR2_ERR_INVALID_ARG, "l2_eps must be finite and >= 0 (got %g)", (double)l2_eps);
    const long long rows = cu_seqlens ? (long long)T : (long long)N * T;
    if (rows * H * d > (1ll << 40)) return fail(GDR2_ERR_INVALID_ARG, "problem too large");
    if ((long long)N * H == 0) return GDR2_OK;
    const bool has_tokens = rows * H > 0;
    if (cu_seqlens && (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) != 0)
        return fail(GDR2_ERR_INVALID_ARG, "cu_seqlens is not 4-byte aligned");
    GDR2_TRY(check_ptr(x, "x", !has_tokens));
    GDR2_TRY(check_ptr(y, "y", !has_tokens));
    if (has_tokens && x == y) return fail(GDR2_ERR_INVALID_ARG, "y must not be x");
    if (!weight && has_tokens) return fail(GDR2_ERR_INVALID_ARG, "weight is NULL");
    if ((reinterpret_cast<uintptr_t>(weight) & 3u) != 0)
        return fail(GDR2_ERR_INVALID_ARG, "weight is not 4-byte aligned");
    GDR2_TRY(check_ptr(state_in, "state_in", true));
    GDR2_TRY(check_ptr(state_out, "state_out", true));
    if (state_in && state_in == state_out && (cu_seqlens || T != 1))
        return fail(GDR2_ERR_INVALID_ARG, "state_out may be state_in only for T = 1 without cu_seqlens");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (!has_tokens && !cu_seqlens) {
        // no tokens: the state passes through
        if (state_out && width > 1 && state_out != state_in) {
            const size_t bytes = (size_t)N * (width - 1) * H * d * (dt == GDR2_BF16 ? 2 : 4);
            cudaError_t e = state_in ? cudaMemcpyAsync(state_out, state_in, bytes, cudaMemcpyDeviceToDevice, s)
                                     : cudaMemsetAsync(state_out, 0, bytes, s);
            return launched(e, "gdr2_short_conv_silu (T = 0)");
        }
        return GDR2_OK;
    }
    gdr2::ConvArgs a{N, T, H, d, width, dt == GDR2_BF16, l2norm != 0, l2_eps, cu_seqlens, x, weight,
                     width > 1 ? state_in : nullptr, width > 1 ? state_out : nullptr, y, nullptr};
    GDR2_TRY(device_status(&a.status));
    return launched(gdr2::launch_short_conv(a, s), "gdr2_short_conv_silu");
}

gdr2_status gdr2_gate_activations(gdr2_dtype dt, long long n_alpha, const void *a, float *log_alpha, long long n_b,
                                  const void *b_pre, void *b, long long n_w, const void *w_pre, void *w,
                                  void *stream)
{
    GDR2_TRY(check_dtype(dt));
    if (n_alpha < 0 || n_b < 0 || n_w < 0) return fail(GDR2_ERR_INVALID_ARG, "negative element count");
    const void *ins[3] = {a, b_pre, w_pre};
    const void *outs[3] = {log_alpha, b, w};
    const long long ns[3] = {n_alpha, n_b, n_w};
    const char *names[3] = {"a / log_alpha", "b_pre / b", "w_pre / w"};
    for (int k = 0; k < 3; ++k) {
        if (ns[k] == 0) continue;
        if (!ins[k] != !outs[k]) return fail(GDR2_ERR_INVALID_ARG, "%s: give both or neither", names[k]);
        if (!ins[k]) continue;
        if (!aligned16(ins[k]) || !aligned16(outs[k]))
            return fail(GDR2_ERR_INVALID_ARG, "%s: not 16-byte aligned", names[k]);
        if (ins[k] == outs[k] && k == 0 && dt == GDR2_BF16)
            return fail(GDR2_ERR_INVALID_ARG, "log_alpha (fp32) cannot overwrite a (bf16)");
    }
    gdr2::ActArgs args{dt == GDR2_BF16, a ? n_alpha : 0, b_pre ? n_b : 0, w_pre ? n_w : 0, a, b_pre, w_pre,
                       log_alpha, b, w};
    return launched(gdr2::launch_gate_activations(args, static_cast<cudaStream_t>(stream)), "gdr2_gate_activations");
}

gdr2_status gdr2_segment_states(int B, int G, int H, int dk, int dv, const float *A, const float *Bst,
                                const float *S0, float *S_starts, float *S_T, void *stream)
{
    if (B < 0 || G < 0 || H < 0) return fail(GDR2_ERR_INVALID_ARG, "negative size (B=%d G=%d H=%d)", B, G, H);
    if ((dk != 64 && dk != 128) || (dv != 64 && dv != 128))
        return fail(GDR2_ERR_UNSUPPORTED, "dk and dv must be 64 or 128 (dk=%d dv=%d)", dk, dv);
    if ((long long)B * G * H * dk * (dk > dv ? dk : dv) > (1ll << 40)) return fail(GDR2_ERR_INVALID_ARG, "problem too large");
    if ((long long)B * H == 0) return GDR2_OK;
    const bool segs = G > 0;
    GDR2_TRY(check_ptr(A, "A", !segs));
    GDR2_TRY(check_ptr(Bst, "Bst", !segs));
    GDR2_TRY(check_ptr(S_starts, "S_starts", !segs));
    GDR2_TRY(check_ptr(S0, "S0", true));
    GDR2_TRY(check_ptr(S_T, "S_T", true));
    gdr2::SegArgs a{B, G, H, dk, dv, A, Bst, S0, S_starts, S_T};
    return launched(gdr2::launch_segment_states(a, static_cast<cudaStream_t>(stream)), "gdr2_segment_states");
}

gdr2_status gdr2_decode_step_gated(int N, int H, int dk, int dv, gdr2_dtype dt, int gates, const void *q,
                                   const void *k, const void *v, const float *log_alpha, const void *b,
                                   const void *w, float *S, void *o, void *stream)
{
    GDR2_TRY(check_dims(N, 1, H, dk, dv));
    GDR2_TRY(check_dtype(dt));
    GDR2_TRY(check_gates(gates));
    const bool any = (long long)N * H > 0;
    GDR2_TRY(check_ptr(q, "q", !any));
    GDR2_TRY(check_ptr(k, "k", !any));
    GDR2_TRY(check_ptr(v, "v", !any));
    GDR2_TRY(check_ptr(log_alpha, "log_alpha", !any));
    GDR2_TRY(check_gate_ptr(b, "b", !any, gates & GDR2_GATE_SCALAR_B, dt));
    GDR2_TRY(check_gate_ptr(w, "w", !any, gates & GDR2_GATE_SCALAR_W, dt));
    GDR2_TRY(check_ptr(S, "S", !any));
    GDR2_TRY(check_ptr(o, "o", !any));
    if (!any) return GDR2_OK;
    gdr2::DecodeArgs a{N, H, dk, dv, dt == GDR2_BF16, q, k, v, log_alpha, b, w, S, o, nullptr, gates};
    GDR2_TRY(device_status(&a.status));
    return launched(gdr2::launch_decode(a, static_cast<cudaStream_t>(stream)), "gdr2_decode_step");
}

gdr2_status gdr2_decode_step(int N, int H, int dk, int dv, gdr2_dtype dt, const void *q, const void *k,
                             const void *v, const float *log_alpha, const void *b, const void *w, float *S,
                             void *o, void *stream)
{
    return gdr2_decode_step_gated(N, H, dk, dv, dt, 0, q, k, v, log_alpha, b, w, S, o, stream);
}

size_t gdr2_backward_workspace_bytes(int B, int T, int H, int dk, int dv, gdr2_dtype dt)
{
    if (B < 0 || T < 0 || H < 0 || dk <= 0 || dv <= 0) return 0;
    return gdr2::backward_workspace_bytes(B, T, H, dk, dv, dt == GDR2_BF16);
}

gdr2_status gdr2_backward_gated(int B, int T, int H, int dk, int dv, gdr2_dtype dt, int gates, const void *q,
                                const void *k, const void *v, const float *log_alpha, const void *b, const void *w,
                                const float *S0, const void *dO, const float *dS_T, const float *saved_states,
                                void *dq, void *dk_, void *dv_, float *dlog_alpha, void *db, void *dw, float *dS0,
                                void *workspace, size_t workspace_bytes, void *stream)
{
    GDR2_TRY(check_dims(B, T, H, dk, dv));
    GDR2_TRY(check_dtype(dt));
    GDR2_TRY(check_gates(gates));
    if (gates && !(dt == GDR2_BF16 && dk == 128 && dv == 128))
        return fail(GDR2_ERR_UNSUPPORTED, "scalar gates in the backward need bf16 inputs with dk = dv = 128");
    const bool has_tokens = (long long)B * T * H > 0;
    const char *names[] = {"q", "k", "v", "log_alpha", "dO", "dq", "dk", "dv", "dlog_alpha"};
    const void *ptrs[] = {q, k, v, log_alpha, dO, dq, dk_, dv_, dlog_alpha};
    for (int i = 0; i < 9; ++i) GDR2_TRY(check_ptr(ptrs[i], names[i], !has_tokens));
    GDR2_TRY(check_gate_ptr(b, "b", !has_tokens, gates & GDR2_GATE_SCALAR_B, dt));
    GDR2_TRY(check_gate_ptr(db, "db", !has_tokens, gates & GDR2_GATE_SCALAR_B, dt));
    GDR2_TRY(check_gate_ptr(w, "w", !has_tokens, gates & GDR2_GATE_SCALAR_W, dt));
    GDR2_TRY(check_gate_ptr(dw, "dw", !has_tokens, gates & GDR2_GATE_SCALAR_W, dt));
    GDR2_TRY(check_ptr(S0, "S0", true));
    GDR2_TRY(check_ptr(dS_T, "dS_T", true));
    GDR2_TRY(check_ptr(saved_states, "saved_states", true));
    GDR2_TRY(check_ptr(dS0, "dS0", true));
    if ((long long)B * H == 0) return GDR2_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (T == 0) {
        if (dS0) {
            const size_t bytes = (size_t)B * H * dk * dv * sizeof(float);
            cudaError_t e = dS_T ? cudaMemcpyAsync(dS0, dS_T, bytes, cudaMemcpyDeviceToDevice, s)
                                 : cudaMemsetAsync(dS0, 0, bytes, s);
            return launched(e, "gdr2_backward (T = 0)");
        }
        return GDR2_OK;
    }
    const size_t need = gdr2::backward_workspace_bytes(B, T, H, dk, dv, dt == GDR2_BF16);
    if (!workspace || workspace_bytes < need)
        return fail(GDR2_ERR_INVALID_ARG, "workspace too small: %zu bytes given, %zu needed", workspace_bytes, need);
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return fail(GDR2_ERR_INVALID_ARG, "workspace is not 256-byte aligned");
    gdr2::BwdArgs a{B, T, H, dk, dv, dt == GDR2_BF16, q, k, v, log_alpha, b, w, S0, dO, dS_T, saved_states,
                    dq, dk_, dv_, dlog_alpha, db, dw, dS0, workspace, workspace_bytes, nullptr, gates};
    GDR2_TRY(device_status(&a.status));
    if (gates && !gdr2::backward_tc_supported(a))
        return fail(GDR2_ERR_UNSUPPORTED, "scalar gates in the backward need the tensor-core path (no driver entry)");
    return launched(gdr2::launch_backward(a, s), "gdr2_backward");
}

gdr2_status gdr2_backward(int B, int T, int H, int dk, int dv, gdr2_dtype dt, const void *q, const void *k,
                          const void *v, const float *log_alpha, const void *b, const void *w, const float *S0,
                          const void *dO, const float *dS_T, const float *saved_states, void *dq, void *dk_,
                          void *dv_, float *dlog_alpha, void *db, void *dw, float *dS0, void *workspace,
                          size_t workspace_bytes, void *stream)
{
    return gdr2_backward_gated(B, T, H, dk, dv, dt, 0, q, k, v, log_alpha, b, w, S0, dO, dS_T, saved_states, dq,
                               dk_, dv_, dlog_alpha, db, dw, dS0, workspace, workspace_bytes, stream);
}

gdr2_status gdr2_backward_noalloc(int B, int T, int H, int dk, int dv, gdr2_dtype dt, const void *q, const void *k,
                                  const void *v, const float *log_alpha, const void *b, const void *w,
                                  const float *S0, const void *dO, const float *dS_T, const float *saved_states,
                                  void *dq, void *dk_, void *dv_, float *dlog_alpha, void *db, void *dw, float *dS0,
                                  void *stream)
{
    GDR2_TRY(check_dims(B, T, H, dk, dv));
    GDR2_TRY(check_dtype(dt));
    const bool has_tokens = (long long)B * T * H > 0;
    const char *names[] = {"q", "k", "v", "log_alpha", "b", "w", "dO", "dq", "dk", "dv", "dlog_alpha", "db", "dw"};
    const void *ptrs[] = {q, k, v, log_alpha, b, w, dO, dq, dk_, dv_, dlog_alpha, db, dw};
    for (int i = 0; i < 13; ++i) GDR2_TRY(check_ptr(ptrs[i], names[i], !has_tokens));
    GDR2_TRY(check_ptr(S0, "S0", true));
    GDR2_TRY(check_ptr(dS_T, "dS_T", true));
    GDR2_TRY(check_ptr(saved_states, "saved_states", true));
    GDR2_TRY(check_ptr(dS0, "dS0", true));
    if ((long long)B * H == 0) return GDR2_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (T == 0) {
        if (dS0) {
            const size_t bytes = (size_t)B * H * dk * dv * sizeof(float);
            cudaError_t e = dS_T ? cudaMemcpyAsync(dS0, dS_T, bytes, cudaMemcpyDeviceToDevice, s)
                                 : cudaMemsetAsync(dS0, 0, bytes, s);
            return launched(e, "gdr2_backward_noalloc (T = 0)");
        }
        return GDR2_OK;
    }
    const size_t need = gdr2::backward_noalloc_scratch_needed(B, T, H, dk, dv, saved_states != nullptr);
    if (need > GDR2_NOALLOC_SCRATCH_BYTES)
        return fail(GDR2_ERR_UNSUPPORTED,
                    "gdr2_backward_noalloc: this problem needs %zu bytes of scratch but the built-in array holds "
                    "%zu (GDR2_NOALLOC_SCRATCH_BYTES); pass saved_states, split the batch, or use gdr2_backward",
                    need, (size_t)GDR2_NOALLOC_SCRATCH_BYTES);
    gdr2::BwdArgs a{B, T, H, dk, dv, dt == GDR2_BF16, q, k, v, log_alpha, b, w, S0, dO, dS_T, saved_states,
                    dq, dk_, dv_, dlog_alpha, db, dw, dS0, nullptr, 0, nullptr};
    GDR2_TRY(device_status(&a.status));
    return launched(gdr2::launch_backward_noalloc(a, s), "gdr2_backward_noalloc");
}

gdr2_status gdr2_sync_status(void *stream)
{
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return fail(GDR2_ERR_CUDA, "cudaStreamSynchronize: %s", cudaGetErrorString(e));
    unsigned *dev_word = nullptr;
    GDR2_TRY(device_status(&dev_word));
    unsigned word = 0;
    e = cudaMemcpyFromSymbolAsync(&word, g_status_word, sizeof(word), 0, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(dev_word, 0, sizeof(unsigned), s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return fail(GDR2_ERR_CUDA, "reading the status word: %s", cudaGetErrorString(e));
    if (word & gdr2::kStatusTimeout)
        return fail(GDR2_ERR_TIMEOUT, "a kernel gave up a bounded device wait (status 0x%x)", word);
    if (word & gdr2::kStatusBadSeqlens)
        return fail(GDR2_ERR_INVALID_ARG,
                    "cu_seqlens was not a nondecreasing sequence from 0 to T; that call computed nothing");
    g_last_error[0] = '\0';
    return GDR2_OK;
}

}  // extern "C"
