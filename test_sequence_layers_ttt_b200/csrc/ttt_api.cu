// Host layer of the C ABI declared in include/ttt.h: argument validation,
// kernel-family dispatch and status mapping.  Validation runs entirely on the
// host and launches nothing when it fails.
#include <climits>
#include <cstdint>
#include <cstdlib>
#include <cstring>

#include "ttt_internal.h"

namespace ttt {
// TTT-MLP decode with the running state in registers (d = 64, hidden = 256),
// in place on W*_T / b*_T and W*_mb / b*_mb (ttt_mlp_decode.cu).
bool mlp_decode_supports(const MlpArgs& a);
cudaError_t launch_mlp_decode(const MlpArgs& a, cudaStream_t stream);
}  // namespace ttt

namespace {

using ttt::LinearArgs;
using ttt::MlpArgs;

struct Span {
    const void* p;
    size_t bytes;
};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlap(Span a, Span b) {
    if (!a.p || !b.p || a.bytes == 0 || b.bytes == 0) return false;
    uintptr_t a0 = reinterpret_cast<uintptr_t>(a.p), b0 = reinterpret_cast<uintptr_t>(b.p);
    return a0 < b0 + b.bytes && b0 < a0 + a.bytes;
}

bool check_env() {
    static const bool on = [] {
        const char* v = std::getenv("TTT_CHECK");
        return v && v[0] && std::strcmp(v, "0") != 0;
    }();
    // the fault-injection hook makes a launch abandon its waits: report that as a status
    return on || ttt::drop_chunk_hook() >= 0;
}

// In check mode the device error words are cleared before the launch, so the
// status a checked call returns reflects that call alone (calls overlapping on
// several streams still share the words).
bool prepare() {
    if (!check_env()) return true;
    unsigned int stale = 0;
    return ttt::read_and_clear_device_error(&stale) == cudaSuccess &&
           ttt::read_and_clear_mlp_error(&stale) == cudaSuccess &&
           ttt::read_and_clear_umma_error(&stale) == cudaSuccess &&
           ttt::read_and_clear_prologue_error(&stale) == cudaSuccess;
}

bool valid_mini_batch(int mb) { return mb >= 1 && (mb % 16 == 0 || mb == 1 || mb == 2 || mb == 4 || mb == 8); }

// Outputs must not overlap any other buffer, except that an output state
// buffer may be exactly its initial-state buffer (in-place update).
ttt_status check_aliasing(const Span* outs, int n_out, const Span* ins, const int* same_as, int n_in) {
    for (int o = 0; o < n_out; o++) {
        for (int i = 0; i < n_in; i++) {
            if (same_as[o] == i && outs[o].p == ins[i].p) continue;
            if (overlap(outs[o], ins[i])) return TTT_ERR_ALIAS;
        }
        for (int o2 = o + 1; o2 < n_out; o2++)
            if (overlap(outs[o], outs[o2])) return TTT_ERR_ALIAS;
    }
    return TTT_OK;
}

ttt_status finish(cudaError_t launch, cudaStream_t stream) {
    if (launch != cudaSuccess) return TTT_ERR_CUDA;
    if (!check_env()) return TTT_OK;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return TTT_ERR_CUDA;
    unsigned int flag = 0, mlp_flag = 0, umma_flag = 0, pro_flag = 0;
    if (ttt::read_and_clear_device_error(&flag) != cudaSuccess) return TTT_ERR_CUDA;
    if (ttt::read_and_clear_mlp_error(&mlp_flag) != cudaSuccess) return TTT_ERR_CUDA;
    if (ttt::read_and_clear_umma_error(&umma_flag) != cudaSuccess) return TTT_ERR_CUDA;
    if (ttt::read_and_clear_prologue_error(&pro_flag) != cudaSuccess) return TTT_ERR_CUDA;
    return (flag | mlp_flag | umma_flag | pro_flag) ? TTT_ERR_TIMEOUT : TTT_OK;
}

ttt_status validate_linear(const LinearArgs& a) {
    if (a.B < 1 || a.H < 1 || a.T < 0 || (long long)a.B * a.H > INT_MAX) return TTT_ERR_SHAPE;
    if (!valid_mini_batch(a.mini_batch)) return TTT_ERR_SHAPE;
    if (a.dtype != TTT_BF16 && a.dtype != TTT_F32) return TTT_ERR_DTYPE;
    if (a.mode != TTT_LN_RESIDUAL && a.mode != TTT_PLAIN) return TTT_ERR_UNSUPPORTED;
    if (a.d != 16 && a.d != 32 && a.d != 64) return TTT_ERR_UNSUPPORTED;
    const bool ln = a.mode == TTT_LN_RESIDUAL;
    if (ln && !(a.ln_eps > 0.f)) return TTT_ERR_SHAPE;
    // with T == 0 the token buffers are empty and may be NULL
    if (a.T > 0 && (!a.Q || !a.K || !a.V || !a.eta || !a.Z)) return TTT_ERR_NULL;
    if (!a.W0 || !a.W_T) return TTT_ERR_NULL;
    if (ln && (!a.b0 || !a.gamma || !a.beta || !a.b_T)) return TTT_ERR_NULL;
    const void* ptrs[] = {a.Q, a.K, a.V, a.eta, a.W0, a.b0, a.gamma, a.beta, a.Z, a.W_T, a.b_T};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return TTT_ERR_ALIGN;

    const size_t es = a.dtype == TTT_BF16 ? 2 : 4;
    const size_t bh = (size_t)a.B * a.H, ntok = bh * (size_t)a.T, d = a.d;
    Span ins[] = {{a.Q, ntok * d * es},   {a.K, ntok * d * es},      {a.V, ntok * d * es},
                  {a.eta, ntok * 4},      {a.W0, bh * d * d * 4},    {a.b0, a.b0 ? bh * d * 4 : 0},
                  {a.gamma, a.gamma ? (size_t)a.H * d * 4 : 0},      {a.beta, a.beta ? (size_t)a.H * d * 4 : 0}};
    Span outs[] = {{a.Z, ntok * d * 4}, {a.W_T, bh * d * d * 4}, {a.b_T, a.b_T ? bh * d * 4 : 0}};
    const int same_as[] = {-1, 4, 5};
    return check_aliasing(outs, 3, ins, same_as, 8);
}

// Decode: the forward scan's checks, plus the position and the mini-batch start
// state (W_mb, b_mb), which is read and written in place like W and b.
ttt_status validate_decode(const LinearArgs& a) {
    ttt_status st = validate_linear(a);
    if (st != TTT_OK) return st;
    if (a.pos0 < 0 || a.pos0 >= a.mini_batch) return TTT_ERR_SHAPE;
    const bool ln = a.mode == TTT_LN_RESIDUAL;
    if (!a.Wm_T || (ln && !a.bm_T)) return TTT_ERR_NULL;
    if (!aligned16(a.Wm_T) || (a.bm_T && !aligned16(a.bm_T))) return TTT_ERR_ALIGN;
    const size_t es = a.dtype == TTT_BF16 ? 2 : 4;
    const size_t bh = (size_t)a.B * a.H, ntok = bh * (size_t)a.T, d = a.d;
    const size_t bbytes = ln ? bh * d * 4 : 0;
    Span ins[] = {{a.Q, ntok * d * es}, {a.K, ntok * d * es}, {a.V, ntok * d * es}, {a.eta, ntok * 4},
                  {a.gamma, a.gamma ? (size_t)a.H * d * 4 : 0}, {a.beta, a.beta ? (size_t)a.H * d * 4 : 0}};
    Span outs[] = {{a.Z, ntok * d * 4}, {a.W_T, bh * d * d * 4}, {a.b_T, a.b_T ? bbytes : 0},
                   {a.Wm_T, bh * d * d * 4}, {a.bm_T, a.bm_T ? bbytes : 0}};
    const int same_as[] = {-1, -1, -1, -1, -1};
    return check_aliasing(outs, 5, ins, same_as, 6);
}

ttt_status validate_mlp(const MlpArgs& a) {
    if (a.B < 1 || a.H < 1 || a.T < 0 || (long long)a.B * a.H > INT_MAX) return TTT_ERR_SHAPE;
    if (!valid_mini_batch(a.mini_batch)) return TTT_ERR_SHAPE;
    if (a.dtype != TTT_BF16 && a.dtype != TTT_F32) return TTT_ERR_DTYPE;
    if (!ttt::mlp_generic_supports(a)) return TTT_ERR_UNSUPPORTED;
    if (!(a.ln_eps > 0.f)) return TTT_ERR_SHAPE;
    const void* req[] = {a.Q, a.K, a.V, a.eta, a.Z, a.W1_0, a.b1_0, a.W2_0, a.b2_0, a.gamma,
                         a.beta, a.W1_T, a.b1_T, a.W2_T, a.b2_T};
    // with T == 0 the token buffers (the first five) are empty and may be NULL
    for (int i = a.T > 0 ? 0 : 5; i < 15; i++)
        if (!req[i]) return TTT_ERR_NULL;
    for (const void* p : req)
        if (p && !aligned16(p)) return TTT_ERR_ALIGN;
    const size_t es = a.dtype == TTT_BF16 ? 2 : 4;
    const size_t bh = (size_t)a.B * a.H, ntok = bh * (size_t)a.T, d = a.d, hd = a.hidden;
    Span ins[] = {{a.Q, ntok * d * es},     {a.K, ntok * d * es},   {a.V, ntok * d * es},
                  {a.eta, ntok * 4},        {a.W1_0, bh * d * hd * 4}, {a.b1_0, bh * hd * 4},
                  {a.W2_0, bh * hd * d * 4}, {a.b2_0, bh * d * 4},   {a.gamma, (size_t)a.H * d * 4},
                  {a.beta, (size_t)a.H * d * 4}};
    Span outs[] = {{a.Z, ntok * d * 4}, {a.W1_T, bh * d * hd * 4}, {a.b1_T, bh * hd * 4},
                   {a.W2_T, bh * hd * d * 4}, {a.b2_T, bh * d * 4}};
    const int same_as[] = {-1, 4, 5, 6, 7};
    return check_aliasing(outs, 5, ins, same_as, 10);
}

// TTT-MLP decode: the forward scan's checks with the running state in place,
// plus the position and the mini-batch start state (read and written in place).
ttt_status validate_mlp_decode(const MlpArgs& a) {
    ttt_status st = validate_mlp(a);
    if (st != TTT_OK) return st;
    if (a.pos0 < 0 || a.pos0 >= a.mini_batch) return TTT_ERR_SHAPE;
    const void* mb[] = {a.W1_mb, a.b1_mb, a.W2_mb, a.b2_mb};
    for (const void* p : mb) {
        if (!p) return TTT_ERR_NULL;
        if (!aligned16(p)) return TTT_ERR_ALIGN;
    }
    const size_t es = a.dtype == TTT_BF16 ? 2 : 4;
    const size_t bh = (size_t)a.B * a.H, ntok = bh * (size_t)a.T, d = a.d, hd = a.hidden;
    Span ins[] = {{a.Q, ntok * d * es}, {a.K, ntok * d * es}, {a.V, ntok * d * es}, {a.eta, ntok * 4},
                  {a.gamma, (size_t)a.H * d * 4}, {a.beta, (size_t)a.H * d * 4}};
    Span outs[] = {{a.Z, ntok * d * 4},     {a.W1_T, bh * d * hd * 4},  {a.b1_T, bh * hd * 4},
                   {a.W2_T, bh * hd * d * 4}, {a.b2_T, bh * d * 4},      {a.W1_mb, bh * d * hd * 4},
                   {a.b1_mb, bh * hd * 4},   {a.W2_mb, bh * hd * d * 4}, {a.b2_mb, bh * d * 4}};
    const int same_as[] = {-1, -1, -1, -1, -1, -1, -1, -1, -1};
    return check_aliasing(outs, 9, ins, same_as, 6);
}

// Layer backward: shapes and modes the backward kernels take, pointers, alignment,
// workspace size and overlaps (every output is distinct from every input, from
// the workspace and from every other output).
ttt_status validate_linear_backward(const ttt::LinearBwdArgs& a, const void* workspace, size_t workspace_bytes) {
    const LinearArgs& f = a.f;
    if (f.B < 1 || f.H < 1 || f.T < 0 || (long long)f.B * f.H > INT_MAX) return TTT_ERR_SHAPE;
    if (!valid_mini_batch(f.mini_batch)) return TTT_ERR_SHAPE;
    if (f.dtype != TTT_BF16 && f.dtype != TTT_F32) return TTT_ERR_DTYPE;
    if (f.mode != TTT_LN_RESIDUAL && f.mode != TTT_PLAIN) return TTT_ERR_UNSUPPORTED;
    if (!(f.ln_eps > 0.f)) return TTT_ERR_SHAPE;
    if (!ttt::linear_backward_supports(a)) return TTT_ERR_UNSUPPORTED;
    if (f.T > 0 && (!f.Q || !f.K || !f.V || !f.eta || !a.dZ || !a.dQ || !a.dK || !a.dV || !a.deta))
        return TTT_ERR_NULL;
    if (!f.W0 || !f.b0 || !f.gamma || !f.beta || !a.dW0 || !a.db0 || !a.dgamma || !a.dbeta) return TTT_ERR_NULL;
    const void* ptrs[] = {f.Q, f.K, f.V, f.eta, f.W0, f.b0, f.gamma, f.beta, a.dZ, a.dW_T, a.db_T, a.dQ,
                          a.dK, a.dV, a.deta, a.dW0, a.db0, a.dgamma, a.dbeta, workspace};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return TTT_ERR_ALIGN;
    const size_t need = ttt::linear_backward_workspace_bytes(f.B, f.H, f.T, f.d, f.mini_batch);
    if (!workspace || workspace_bytes < need) return TTT_ERR_WORKSPACE;
    const size_t es = f.dtype == TTT_BF16 ? 2 : 4;
    const size_t bh = (size_t)f.B * f.H, ntok = bh * (size_t)f.T, d = f.d;
    Span ins[] = {{f.Q, ntok * d * es},      {f.K, ntok * d * es},         {f.V, ntok * d * es},
                  {f.eta, ntok * 4},         {f.W0, bh * d * d * 4},       {f.b0, bh * d * 4},
                  {f.gamma, (size_t)f.H * d * 4}, {f.beta, (size_t)f.H * d * 4}, {a.dZ, ntok * d * 4},
                  {a.dW_T, a.dW_T ? bh * d * d * 4 : 0}, {a.db_T, a.db_T ? bh * d * 4 : 0}, {workspace, need}};
    Span outs[] = {{a.dQ, ntok * d * 4}, {a.dK, ntok * d * 4},   {a.dV, ntok * d * 4},
                   {a.deta, ntok * 4},   {a.dW0, bh * d * d * 4}, {a.db0, bh * d * 4},
                   {a.dgamma, (size_t)f.H * d * 4}, {a.dbeta, (size_t)f.H * d * 4}};
    const int same_as[] = {-1, -1, -1, -1, -1, -1, -1, -1};
    return check_aliasing(outs, 8, ins, same_as, 12);
}

ttt_status validate_prologue(const ttt::PrologueArgs& a) {
    if (a.B < 1 || a.T < 1 || a.H < 1 || a.d_model < 1 || (long long)a.B * a.T >= (1LL << 31)) return TTT_ERR_SHAPE;
    if (!(a.rope_base > 1.f) || !(a.eta_base == a.eta_base)) return TTT_ERR_SHAPE;
    if (!ttt::prologue_supports(a.B, a.T, a.H, a.d, a.d_model)) return TTT_ERR_UNSUPPORTED;
    const void* req[] = {a.x, a.theta_q, a.theta_k, a.theta_v, a.theta_lr, a.b_lr, a.Q, a.K, a.V, a.eta};
    for (const void* p : req)
        if (!p) return TTT_ERR_NULL;
    for (const void* p : req)
        if (!aligned16(p)) return TTT_ERR_ALIGN;
    const size_t tok = (size_t)a.B * a.T, hd = (size_t)a.H * a.d, w = (size_t)a.d_model * hd * 2;
    Span ins[] = {{a.x, tok * a.d_model * 2}, {a.theta_q, w}, {a.theta_k, w}, {a.theta_v, w},
                  {a.theta_lr, (size_t)a.H * a.d_model * 2}, {a.b_lr, (size_t)a.H * 4}};
    Span outs[] = {{a.Q, tok * hd * 2}, {a.K, tok * hd * 2}, {a.V, tok * hd * 2}, {a.eta, tok * a.H * 4}};
    const int same_as[] = {-1, -1, -1, -1};
    return check_aliasing(outs, 4, ins, same_as, 6);
}

}  // namespace

extern "C" {

ttt_status ttt_prologue_forward(int B, int T, int H, int d, int d_model, int pos0, float eta_base,
                                float rope_base, int rotary, const void* x, const void* theta_q,
                                const void* theta_k, const void* theta_v, const void* theta_lr,
                                const float* b_lr, void* Q, void* K, void* V, float* eta,
                                ttt_stream_t stream) {
    ttt::PrologueArgs a{B, T, H, d, d_model, pos0, rotary ? 1 : 0, eta_base, rope_base, x, theta_q, theta_k,
                        theta_v, theta_lr, b_lr, Q, K, V, eta};
    ttt_status st = validate_prologue(a);
    if (st != TTT_OK) return st;
    if (!prepare()) return TTT_ERR_CUDA;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    return finish(ttt::launch_prologue(a, s), s);
}

size_t ttt_linear_backward_workspace_size(int B, int H, int T, int d, int mini_batch) {
    return ttt::linear_backward_workspace_bytes(B, H, T, d, mini_batch);
}

ttt_status ttt_linear_backward(int B, int H, int T, int d, int mini_batch, ttt_dtype qkv_dtype, ttt_mode mode,
                               float ln_eps, const void* Q, const void* K, const void* V, const float* eta,
                               const float* W0, const float* b0, const float* ln_gamma, const float* ln_beta,
                               const float* dZ, const float* dW_T, const float* db_T, float* dQ, float* dK,
                               float* dV, float* deta, float* dW0, float* db0, float* dgamma, float* dbeta,
                               void* workspace, size_t workspace_bytes, ttt_stream_t stream) {
    ttt::LinearBwdArgs a{};
    a.f = LinearArgs{B, H, T, d, mini_batch, qkv_dtype, mode, ln_eps, Q, K, V, eta, W0, b0, ln_gamma, ln_beta,
                     nullptr, nullptr, nullptr};
    a.dZ = dZ;
    a.dW_T = dW_T;
    a.db_T = db_T;
    a.dQ = dQ;
    a.dK = dK;
    a.dV = dV;
    a.deta = deta;
    a.dW0 = dW0;
    a.db0 = db0;
    a.dgamma = dgamma;
    a.dbeta = dbeta;
    ttt_status st = validate_linear_backward(a, workspace, workspace_bytes);
    if (st != TTT_OK) return st;
    if (!prepare()) return TTT_ERR_CUDA;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    return finish(ttt::launch_linear_backward(a, static_cast<float*>(workspace), s), s);
}


ttt_status ttt_linear_forward_impl(int B, int H, int T, int d, int mini_batch, ttt_dtype qkv_dtype,
                                   ttt_mode mode, float ln_eps, const void* Q, const void* K,
                                   const void* V, const float* eta, const float* W0,
                                   const float* b0, const float* ln_gamma, const float* ln_beta,
                                   float* Z, float* W_T, float* b_T, ttt_impl impl,
                                   ttt_stream_t stream) {
    LinearArgs a{B, H, T, d, mini_batch, qkv_dtype, mode, ln_eps, Q, K, V, eta,
                 W0, b0, ln_gamma, ln_beta, Z, W_T, b_T};
    ttt_status st = validate_linear(a);
    if (st != TTT_OK) return st;
    if (!prepare()) return TTT_ERR_CUDA;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    switch (impl) {
        case TTT_IMPL_AUTO:
            if (ttt::linear_tc_supports(a)) return finish(ttt::launch_linear_tc(a, s), s);
            return finish(ttt::launch_linear_generic(a, s), s);
        case TTT_IMPL_GENERIC:
            return finish(ttt::launch_linear_generic(a, s), s);
        case TTT_IMPL_TENSORCORE:
            if (!ttt::linear_tc_supports(a)) return TTT_ERR_UNSUPPORTED;
            return finish(ttt::launch_linear_tc(a, s), s);
        case TTT_IMPL_TCGEN05:
            if (!ttt::linear_umma_supports(a)) return TTT_ERR_UNSUPPORTED;
            return finish(ttt::launch_linear_umma(a, s), s);
        default:
            return TTT_ERR_UNSUPPORTED;
    }
}

ttt_impl ttt_linear_pick_impl(int B, int H, int T, int d, int mini_batch, ttt_dtype qkv_dtype,
                              ttt_mode mode) {
    LinearArgs a{B, H, T, d, mini_batch, qkv_dtype, mode, 1e-6f, nullptr, nullptr, nullptr,
                 nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr};
    if (ttt::linear_tc_supports(a)) return TTT_IMPL_TENSORCORE;
    return ttt::linear_generic_supports(a) ? TTT_IMPL_GENERIC : TTT_IMPL_AUTO;
}

ttt_status ttt_linear_forward(int B, int H, int T, int d, int mini_batch, ttt_dtype qkv_dtype,
                              ttt_mode mode, float ln_eps, const void* Q, const void* K,
                              const void* V, const float* eta, const float* W0, const float* b0,
                              const float* ln_gamma, const float* ln_beta, float* Z, float* W_T,
                              float* b_T, ttt_stream_t stream) {
    return ttt_linear_forward_impl(B, H, T, d, mini_batch, qkv_dtype, mode, ln_eps, Q, K, V, eta,
                                   W0, b0, ln_gamma, ln_beta, Z, W_T, b_T, TTT_IMPL_AUTO, stream);
}

// The family TTT_IMPL_AUTO runs for valid TTT-MLP arguments (TTT_IMPL_AUTO if none covers them)
static ttt_impl mlp_auto_impl(const MlpArgs& a) {
    if (ttt::mlp_split_supports(a) && (long)a.B * a.H <= ttt::kMlpSplitMaxScans) return TTT_IMPL_TENSORCORE_SPLIT;
    if (ttt::mlp_tc_supports(a)) return TTT_IMPL_TENSORCORE;
    return ttt::mlp_generic_supports(a) ? TTT_IMPL_GENERIC : TTT_IMPL_AUTO;
}

ttt_status ttt_linear_decode(int B, int H, int T, int d, int mini_batch, int pos0, ttt_dtype qkv_dtype,
                             ttt_mode mode, float ln_eps, const void* Q, const void* K, const void* V,
                             const float* eta, float* W, float* b, float* W_mb, float* b_mb,
                             const float* ln_gamma, const float* ln_beta, float* Z, ttt_stream_t stream) {
    const bool ln = mode == TTT_LN_RESIDUAL;
    LinearArgs a{B, H, T, d, mini_batch, qkv_dtype, mode, ln_eps, Q, K, V, eta, W, ln ? b : nullptr,
                 ln_gamma, ln_beta, Z, W, ln ? b : nullptr,
                 pos0, pos0 > 0 ? W_mb : nullptr, (pos0 > 0 && ln) ? b_mb : nullptr, W_mb, ln ? b_mb : nullptr};
    ttt_status st = validate_decode(a);
    if (st != TTT_OK) return st;
    if (!prepare()) return TTT_ERR_CUDA;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (ttt::linear_decode_supports(a)) return finish(ttt::launch_linear_decode(a, s), s);
    return finish(ttt::launch_linear_generic(a, s), s);
}

ttt_status ttt_mlp_forward_impl(int B, int H, int T, int d, int hidden, int mini_batch,
                                ttt_dtype qkv_dtype, float ln_eps, const void* Q, const void* K,
                                const void* V, const float* eta, const float* W1_0, const float* b1_0,
                                const float* W2_0, const float* b2_0, const float* ln_gamma,
                                const float* ln_beta, float* Z, float* W1_T, float* b1_T, float* W2_T,
                                float* b2_T, ttt_impl impl, ttt_stream_t stream) {
    MlpArgs a{B, H, T, d, hidden, mini_batch, qkv_dtype, ln_eps, Q, K, V, eta, W1_0, b1_0,
              W2_0, b2_0, ln_gamma, ln_beta, Z, W1_T, b1_T, W2_T, b2_T};
    ttt_status st = validate_mlp(a);
    if (st != TTT_OK) return st;
    if (!prepare()) return TTT_ERR_CUDA;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (impl == TTT_IMPL_AUTO) impl = mlp_auto_impl(a);
    switch (impl) {
        case TTT_IMPL_GENERIC:
            return finish(ttt::launch_mlp_generic(a, s), s);
        case TTT_IMPL_TENSORCORE:
            if (!ttt::mlp_tc_supports(a)) return TTT_ERR_UNSUPPORTED;
            return finish(ttt::launch_mlp_tc(a, s), s);
        case TTT_IMPL_TENSORCORE_SPLIT:
            if (!ttt::mlp_split_supports(a)) return TTT_ERR_UNSUPPORTED;
            return finish(ttt::launch_mlp_split(a, s), s);
        default:
            return TTT_ERR_UNSUPPORTED;
    }
}

ttt_status ttt_mlp_decode_impl(int B, int H, int T, int d, int hidden, int mini_batch, int pos0,
                               ttt_dtype qkv_dtype, float ln_eps, const void* Q, const void* K, const void* V,
                               const float* eta, float* W1, float* b1, float* W2, float* b2, float* W1_mb,
                               float* b1_mb, float* W2_mb, float* b2_mb, const float* ln_gamma,
                               const float* ln_beta, float* Z, ttt_impl impl, ttt_stream_t stream) {
    MlpArgs a{B, H, T, d, hidden, mini_batch, qkv_dtype, ln_eps, Q, K, V, eta, W1, b1, W2, b2,
              ln_gamma, ln_beta, Z, W1, b1, W2, b2, pos0, W1_mb, b1_mb, W2_mb, b2_mb};
    ttt_status st = validate_mlp_decode(a);
    if (st != TTT_OK) return st;
    if (!prepare()) return TTT_ERR_CUDA;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    switch (impl) {
        case TTT_IMPL_AUTO:
            if (ttt::mlp_decode_supports(a)) return finish(ttt::launch_mlp_decode(a, s), s);
            return finish(ttt::launch_mlp_generic(a, s), s);
        case TTT_IMPL_GENERIC:
            return finish(ttt::launch_mlp_generic(a, s), s);
        default:
            return TTT_ERR_UNSUPPORTED;
    }
}

ttt_status ttt_mlp_decode(int B, int H, int T, int d, int hidden, int mini_batch, int pos0,
                          ttt_dtype qkv_dtype, float ln_eps, const void* Q, const void* K, const void* V,
                          const float* eta, float* W1, float* b1, float* W2, float* b2, float* W1_mb,
                          float* b1_mb, float* W2_mb, float* b2_mb, const float* ln_gamma,
                          const float* ln_beta, float* Z, ttt_stream_t stream) {
    return ttt_mlp_decode_impl(B, H, T, d, hidden, mini_batch, pos0, qkv_dtype, ln_eps, Q, K, V, eta, W1, b1,
                               W2, b2, W1_mb, b1_mb, W2_mb, b2_mb, ln_gamma, ln_beta, Z, TTT_IMPL_AUTO, stream);
}

ttt_impl ttt_mlp_pick_impl(int B, int H, int T, int d, int hidden, int mini_batch, ttt_dtype qkv_dtype) {
    MlpArgs a{B, H, T, d, hidden, mini_batch, qkv_dtype, 1e-6f, nullptr, nullptr, nullptr, nullptr,
              nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr,
              nullptr};
    return mlp_auto_impl(a);
}

ttt_status ttt_mlp_forward(int B, int H, int T, int d, int hidden, int mini_batch,
                           ttt_dtype qkv_dtype, float ln_eps, const void* Q, const void* K,
                           const void* V, const float* eta, const float* W1_0, const float* b1_0,
                           const float* W2_0, const float* b2_0, const float* ln_gamma,
                           const float* ln_beta, float* Z, float* W1_T, float* b1_T, float* W2_T,
                           float* b2_T, ttt_stream_t stream) {
    return ttt_mlp_forward_impl(B, H, T, d, hidden, mini_batch, qkv_dtype, ln_eps, Q, K, V, eta, W1_0,
                                b1_0, W2_0, b2_0, ln_gamma, ln_beta, Z, W1_T, b1_T, W2_T, b2_T,
                                TTT_IMPL_AUTO, stream);
}

ttt_status ttt_linear_backward_static(int B, int H, int T, int d, int mini_batch, ttt_dtype qkv_dtype,
                                      ttt_mode mode, float ln_eps, const void* Q, const void* K, const void* V,
                                      const float* eta, const float* W0, const float* b0, const float* ln_gamma,
                                      const float* ln_beta, const float* dZ, const float* dW_T, const float* db_T,
                                      float* dQ, float* dK, float* dV, float* deta, float* dW0, float* db0,
                                      float* dgamma, float* dbeta, ttt_stream_t stream) {
    // the size check comes first: shapes beyond the fixed array are refused before any CUDA call
    const size_t need = ttt::linear_backward_workspace_bytes(B, H, T, d, mini_batch);
    if (need > ttt::kBackwardStaticWorkspaceBytes) return TTT_ERR_WORKSPACE;
    float* ws = ttt::backward_static_workspace();
    if (!ws) return TTT_ERR_CUDA;
    return ttt_linear_backward(B, H, T, d, mini_batch, qkv_dtype, mode, ln_eps, Q, K, V, eta, W0, b0, ln_gamma,
                               ln_beta, dZ, dW_T, db_T, dQ, dK, dV, deta, dW0, db0, dgamma, dbeta, ws,
                               ttt::kBackwardStaticWorkspaceBytes, stream);
}

const char* ttt_status_string(ttt_status status) {
    switch (status) {
        case TTT_OK: return "TTT_OK";
        case TTT_ERR_NULL: return "TTT_ERR_NULL: a required pointer is NULL";
        case TTT_ERR_SHAPE: return "TTT_ERR_SHAPE: B, H, T, mini_batch or ln_eps out of range";
        case TTT_ERR_DTYPE: return "TTT_ERR_DTYPE: unknown element type";
        case TTT_ERR_ALIGN: return "TTT_ERR_ALIGN: a pointer is not 16-byte aligned";
        case TTT_ERR_ALIAS: return "TTT_ERR_ALIAS: an output overlaps another buffer";
        case TTT_ERR_UNSUPPORTED: return "TTT_ERR_UNSUPPORTED: shape, mode or kernel family not built";
        case TTT_ERR_CUDA: return "TTT_ERR_CUDA: CUDA launch or execution error";
        case TTT_ERR_TIMEOUT: return "TTT_ERR_TIMEOUT: a kernel abandoned a bounded wait";
        case TTT_ERR_WORKSPACE: return "TTT_ERR_WORKSPACE: workspace missing or too small for these arguments";
        default: return "TTT_ERR_UNKNOWN";
    }
}

int ttt_abi_version(void) { return 103; }

#ifdef TTT_TIMELINE
// Timeline builds only (not part of the ABI): copy the clock64 stamps of CTA 0
// of the last launch of kernel `which` (0: ttt_linear_lag_kernel, 1: the backward's
// ttt_linear_backward_kernel) into
// out[kTlRoles][kTlChunks][kTlEvents].
int ttt_debug_timeline(int which, long long* out) {
    if (!out) return TTT_ERR_NULL;
    if (cudaDeviceSynchronize() != cudaSuccess) return TTT_ERR_CUDA;
    const cudaError_t e = which == 0   ? ttt::read_lag_timeline(out)
                          : which == 1 ? ttt::read_bwd_timeline(out)
                                       : cudaErrorInvalidValue;
    return e == cudaSuccess ? TTT_OK : TTT_ERR_CUDA;
}
#endif

}  // extern "C"
