// Internal launch interface between the host layer (ttt_api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>

#include "../../include/ttt.h"

namespace ttt {

struct LinearArgs {
    int B, H, T, d, mini_batch;
    ttt_dtype dtype;
    ttt_mode mode;
    float ln_eps;
    const void *Q, *K, *V;
    const float *eta, *W0, *b0, *gamma, *beta;
    float *Z, *W_T, *b_T;
    // decode only (generic family): position of the first token in its
    // mini-batch, and the mini-batch start state in (read when pos0 > 0) and out
    int pos0;
    const float *Wm0, *bm0;
    float *Wm_T, *bm_T;
};

struct MlpArgs {
    int B, H, T, d, hidden, mini_batch;
    ttt_dtype dtype;
    float ln_eps;
    const void *Q, *K, *V;
    const float *eta, *W1_0, *b1_0, *W2_0, *b2_0, *gamma, *beta;
    float *Z, *W1_T, *b1_T, *W2_T, *b2_T;
    // decode only (generic family): position of the first token in its
    // mini-batch, and the mini-batch start state, read when pos0 > 0 and
    // written in place
    int pos0;
    float *W1_mb, *b1_mb, *W2_mb, *b2_mb;
};

bool linear_generic_supports(const LinearArgs& a);
cudaError_t launch_linear_generic(const LinearArgs& a, cudaStream_t stream);

bool linear_tc_supports(const LinearArgs& a);
cudaError_t launch_linear_tc(const LinearArgs& a, cudaStream_t stream);
// The same scan as the checkpoint pass of the layer backward: stores the state at the start of
// every mini-batch (W [in][out], then b; d^2 + d floats per mini-batch and (batch, head)) into
// `states`; writes neither Z nor the final state (a.Z, a.W_T, a.b_T unused).
cudaError_t launch_linear_tc_checkpoints(const LinearArgs& a, float* states, cudaStream_t stream);

// State products on tcgen05 / TMEM, chain on mma.sync (ttt_linear_umma.cu); same shapes as linear_tc.
bool linear_umma_supports(const LinearArgs& a);
cudaError_t launch_linear_umma(const LinearArgs& a, cudaStream_t stream);
cudaError_t read_and_clear_umma_error(unsigned int* out);

// Decode with the state in registers (d = 64); in place on W_T / b_T and Wm_T / bm_T.
bool linear_decode_supports(const LinearArgs& a);
cudaError_t launch_linear_decode(const LinearArgs& a, cudaStream_t stream);

// TTT-Linear layer backward (ttt_linear_backward.cu): the forward arguments plus
// the upstream gradients and the gradient outputs.
struct LinearBwdArgs {
    LinearArgs f;  // Q, K, V, eta, W0, b0, gamma, beta and the shapes (Z, W_T, b_T unused)
    const float *dZ, *dW_T, *db_T;
    float *dQ, *dK, *dV, *deta, *dW0, *db0, *dgamma, *dbeta;
};
// Size of the file-scope workspace of ttt_linear_backward_static (TTT_BACKWARD_STATIC_WORKSPACE_BYTES).
constexpr size_t kBackwardStaticWorkspaceBytes = TTT_BACKWARD_STATIC_WORKSPACE_BYTES;
float* backward_static_workspace();
bool linear_backward_supports(const LinearBwdArgs& a);
size_t linear_backward_workspace_bytes(int B, int H, int T, int d, int mini_batch);
cudaError_t launch_linear_backward(const LinearBwdArgs& a, float* workspace, cudaStream_t stream);

// The layer's prologue (ttt_prologue.cu): projections, learning-rate gate, rotary embedding.
struct PrologueArgs {
    int B, T, H, d, d_model, pos0, rotary;
    float eta_base, rope_base;
    const void *x, *theta_q, *theta_k, *theta_v, *theta_lr;
    const float* b_lr;
    void *Q, *K, *V;
    float* eta;
};
bool prologue_supports(int B, int T, int H, int d, int d_model);
cudaError_t launch_prologue(const PrologueArgs& a, cudaStream_t stream);
cudaError_t read_and_clear_prologue_error(unsigned int* out);

bool mlp_generic_supports(const MlpArgs& a);
cudaError_t launch_mlp_generic(const MlpArgs& a, cudaStream_t stream);

bool mlp_tc_supports(const MlpArgs& a);
cudaError_t launch_mlp_tc(const MlpArgs& a, cudaStream_t stream);

// Hidden units of each scan split over a 2-CTA cluster; same shapes as mlp_tc.
// Preferred while its 2 B H CTAs (one per SM) fit in one wave: a 148-SM B200
// holds 74 such clusters at once (cudaOccupancyMaxActiveClusters).
constexpr int kMlpSplitMaxScans = 74;
bool mlp_split_supports(const MlpArgs& a);
cudaError_t launch_mlp_split(const MlpArgs& a, cudaStream_t stream);
// Error word of the split kernel (a bounded wait on the other CTA gave up).
cudaError_t read_and_clear_mlp_error(unsigned int* out);

// Device-side error word set by kernels that abandon a bounded wait.
cudaError_t read_and_clear_device_error(unsigned int* out);
#ifdef TTT_TIMELINE
cudaError_t read_lag_timeline(long long* out);     // kTlRoles x kTlChunks x kTlEvents stamps
cudaError_t read_bwd_timeline(long long* out);     // the same layout, the backward's reverse sweep
#endif

// Fault-injection hook: the chunk index named by TTT_DEBUG_DROP_CHUNK (read once
// per process), whose loads the tensor-core TTT-Linear producer skips; -1 when unset.
int drop_chunk_hook();

}  // namespace ttt
