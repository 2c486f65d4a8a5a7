// Internal launcher declarations shared by the library's translation units.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <algorithm>

namespace dsc {

// Records the detail string that dsc_last_error() returns on this host thread.
void set_last_error(const char *msg);

// Wait settings for the next tensor-core launch on this host thread: the normal limit
// and no withheld loads, unless dsc_test_arm_wait_timeout() armed the test hook, which
// this call then disarms.
void take_wait_test(unsigned long long *wait_ns, int *withhold_cta);

// Streaming CUDA-core kernels (stream.cu)
void launch_conv_fwd(const void *x, const void *w, void *y, int B, int T, int D, int G, int W,
                     bool bf16, bool is_static, cudaStream_t s);
int static_dw_partials(int B, int T);
void launch_static_bwd(const void *x, const void *w, const void *dy, void *dx, float *part,
                       float *dw, int B, int T, int D, int W, bool bf16, cudaStream_t s);
// Explicit-filter backward in one pass (dx and dw); false: sizes it does not take
bool launch_dyn_bwd(const void *x, const void *w, const void *dy, void *dx, float *dw, int B, int T, int D,
                    int G, int W, bool bf16, cudaStream_t s);

// Decode step (decode.cu)
bool decode_supported(int D, int G, int W, int R);
cudaError_t launch_decode_lowrank(const void *x, const void *z, const void *U, void *state, void *y,
                                  int B, int D, int G, int W, int R, bool bf16, cudaStream_t s);
cudaError_t launch_decode(const void *x, const void *w, void *state, void *y, int B, int D, int G,
                          int W, bool bf16, cudaStream_t s);
// ... on the tensor cores (tc_lowrank.cu): the forward kernel with the sequences as rows
bool tc_decode_lowrank_supported(int B, int D, int G, int W, int R, bool bf16);
cudaError_t launch_tc_decode_lowrank(const void *x, const void *z, const void *U, void *state, void *y, int B,
                                     int D, int G, int W, int R, cudaStream_t s);

// Sequence-shard halo fix-ups (halo.cu)
cudaError_t launch_halo_fwd_lowrank(const void *x, const void *z, const void *U, const void *x_prev, void *y,
                                    int B, int T, int D, int G, int W, int R, bool bf16, cudaStream_t s);
cudaError_t launch_halo_bwd_lowrank(const void *x_prev, const void *z, const void *U, const void *dy,
                                    const void *dy_next, const void *z_next, void *dx, float *dz, float *dU,
                                    int B, int T, int D, int G, int W, int R, bool bf16, cudaStream_t s);

// CUDA-core kernels (simt.cu)
void launch_conv_dx(const void *w, bool w_is_f32, const void *dy, void *dx, int B, int T, int D,
                    int G, int W, bool bf16, bool is_static, cudaStream_t s);
void launch_dyn_dw(const void *x, const void *dy, float *dw, int B, int T, int D, int G, int W,
                   bool bf16, cudaStream_t s);
void launch_lowrank_fwd_simt(const void *x, const void *z, const void *U, void *y, int B, int T,
                             int D, int G, int W, int R, bool bf16, cudaStream_t s);
size_t lowrank_bwd_simt_workspace(int B, int T, int D, int G, int W);
void launch_lowrank_bwd_simt(const void *x, const void *z, const void *U, const void *dy, void *dx,
                             float *dz, float *dU, void *ws, int B, int T, int D, int G, int W,
                             int R, bool bf16, cudaStream_t s);

// Tensor-core (tcgen05) low-rank kernels (tc_lowrank.cu)
bool tc_lowrank_fwd_supported(int B, int T, int D, int G, int W, int R, bool bf16);
bool tc_lowrank_bwd_supported(int B, int T, int D, int G, int W, int R, bool bf16);
unsigned read_device_fault(bool reset);
unsigned read_device_fault_bwd(bool reset);
// cs: RoPE table [T][dh/2][2] (cos, sin) applied to channels [0, n_rot) of y, or null
cudaError_t launch_tc_lowrank_fwd(const void *x, const void *z, const void *U, void *y, int B,
                                  int T, int D, int G, int W, int R, cudaStream_t s,
                                  const float *cs = nullptr, int dh = 0, int n_rot = 0);
size_t tc_lowrank_bwd_workspace(int B, int T, int D, int G, int W, int R);
// cs: RoPE table [T][dh/2][2]; dy is then the gradient of the rotated output
cudaError_t launch_tc_lowrank_bwd(const void *x, const void *z, const void *U, const void *dy,
                                  void *dx, float *dz, float *dU, void *ws, int B, int T, int D,
                                  int G, int W, int R, cudaStream_t s,
                                  const float *cs = nullptr, int dh = 0, int n_rot = 0);

}  // namespace dsc
