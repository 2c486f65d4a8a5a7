// C-ABI host layer of libdsc.so: argument validation, workspace sizing, dispatch to
// the tensor-core or CUDA-core kernels, and status reporting.  No allocation, no
// synchronisation, no exception crosses the boundary.
#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <cstring>

#include "../../include/dsc.h"
#include "internal.h"

#ifndef DSC_DECODE_TC_MIN_B
#define DSC_DECODE_TC_MIN_B 8      // smallest batch whose decode step runs on the tensor cores
                                   // (B200, D=6144: 5.05 us there against 5.12 on CUDA cores;
                                   // at B=1 the CUDA cores win, 4.8 against 5.1 us)
#endif

namespace {

thread_local char g_err[512] = "";

dsc_status_t fail(dsc_status_t st, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
    return st;
}

dsc_status_t ok() {
    g_err[0] = '\0';
    return DSC_OK;
}

dsc_status_t check_launch(const char *what) {
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(DSC_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
    return ok();
}

dsc_status_t check_launch(const char *what, cudaError_t e0) {
    const cudaError_t e = (e0 != cudaSuccess) ? e0 : cudaGetLastError();
    if (e != cudaSuccess) return fail(DSC_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
    return ok();
}

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

struct Dims {
    int B, T, D, G, W, R;
};

// Shared size/dtype checks.  R < 0 means "no low-rank factor".
dsc_status_t check_dims(const char *fn, Dims d, dsc_dtype_t dt) {
    if (dt != DSC_F32 && dt != DSC_BF16) return fail(DSC_ERR_INVALID_ARG, "%s: unknown dtype %d", fn, (int)dt);
    if (d.B <= 0 || d.T <= 0 || d.D <= 0 || d.G <= 0 || d.W <= 0 || (d.R != -1 && d.R <= 0))
        return fail(DSC_ERR_INVALID_ARG, "%s: sizes must be positive (B=%d T=%d D=%d G=%d W=%d R=%d)",
                    fn, d.B, d.T, d.D, d.G, d.W, d.R);
    if (d.D % d.G) return fail(DSC_ERR_INVALID_ARG, "%s: D=%d is not a multiple of G=%d", fn, d.D, d.G);
    if ((long long)d.B * d.T >= (1ll << 31))
        return fail(DSC_ERR_UNSUPPORTED, "%s: B*T=%lld exceeds 2^31-1", fn, (long long)d.B * d.T);
    if (d.W > 8) return fail(DSC_ERR_UNSUPPORTED, "%s: W=%d outside [1,8]", fn, d.W);
    if (d.R > 256) return fail(DSC_ERR_UNSUPPORTED, "%s: R=%d outside [1,256]", fn, d.R);
    const int vec = (dt == DSC_BF16) ? 8 : 4;
    if (d.D % vec)
        return fail(DSC_ERR_UNSUPPORTED, "%s: D=%d must be a multiple of %d for %s", fn, d.D, vec,
                    dt == DSC_BF16 ? "bf16" : "fp32");
    return DSC_OK;
}

dsc_status_t check_ptrs(const char *fn, const void *const *ptrs, const char *const *names, int n) {
    for (int i = 0; i < n; ++i) {
        if (!ptrs[i]) return fail(DSC_ERR_INVALID_ARG, "%s: %s is NULL", fn, names[i]);
        if (!aligned16(ptrs[i])) return fail(DSC_ERR_UNSUPPORTED, "%s: %s is not 16-byte aligned", fn, names[i]);
    }
    return DSC_OK;
}

size_t lowrank_ws(const Dims &d, bool bf16) {
    if (dsc::tc_lowrank_bwd_supported(d.B, d.T, d.D, d.G, d.W, d.R, bf16))
        return dsc::tc_lowrank_bwd_workspace(d.B, d.T, d.D, d.G, d.W, d.R);
    return dsc::lowrank_bwd_simt_workspace(d.B, d.T, d.D, d.G, d.W);
}

}  // namespace

namespace dsc {
void set_last_error(const char *msg) { snprintf(g_err, sizeof(g_err), "%s", msg); }

// Armed wait limit of the test hook for the next tensor-core launch (0: not armed).
thread_local unsigned long long g_test_wait_ns = 0;

void take_wait_test(unsigned long long *wait_ns, int *withhold_cta) {
    if (g_test_wait_ns) {
        *wait_ns = g_test_wait_ns;
        *withhold_cta = 0;
        g_test_wait_ns = 0;
    } else {
        *wait_ns = 1000000000ull;     // one second, as the kernels' own default
        *withhold_cta = -1;
    }
}
}  // namespace dsc

extern "C" {

DSC_API dsc_status_t dsc_fwd(const void *x, const void *w, void *y, int B, int T, int D, int G, int W,
                     dsc_dtype_t dt, dsc_stream_t stream) {
    const char *fn = "dsc_fwd";
    dsc_status_t st = check_dims(fn, Dims{B, T, D, G, W, -1}, dt);
    if (st != DSC_OK) return st;
    const void *p[] = {x, w, y};
    const char *n[] = {"x", "w", "y"};
    if ((st = check_ptrs(fn, p, n, 3)) != DSC_OK) return st;
    dsc::launch_conv_fwd(x, w, y, B, T, D, G, W, dt == DSC_BF16, false, (cudaStream_t)stream);
    return check_launch(fn);
}

DSC_API dsc_status_t dsc_fwd_lowrank(const void *x, const void *z, const void *U, void *y, int B, int T,
                             int D, int G, int W, int R, dsc_dtype_t dt, dsc_stream_t stream) {
    const char *fn = "dsc_fwd_lowrank";
    dsc_status_t st = check_dims(fn, Dims{B, T, D, G, W, R}, dt);
    if (st != DSC_OK) return st;
    const void *p[] = {x, z, U, y};
    const char *n[] = {"x", "z", "U", "y"};
    if ((st = check_ptrs(fn, p, n, 4)) != DSC_OK) return st;
    const bool bf16 = dt == DSC_BF16;
    if (dsc::tc_lowrank_fwd_supported(B, T, D, G, W, R, bf16))
        return check_launch(fn, dsc::launch_tc_lowrank_fwd(x, z, U, y, B, T, D, G, W, R, (cudaStream_t)stream));
    dsc::launch_lowrank_fwd_simt(x, z, U, y, B, T, D, G, W, R, bf16, (cudaStream_t)stream);
    return check_launch(fn);
}

DSC_API size_t dsc_bwd_lowrank_workspace_bytes(int B, int T, int D, int G, int W, int R, dsc_dtype_t dt) {
    if (check_dims("dsc_bwd_lowrank_workspace_bytes", Dims{B, T, D, G, W, R}, dt) != DSC_OK) return 0;
    return lowrank_ws(Dims{B, T, D, G, W, R}, dt == DSC_BF16);
}

DSC_API dsc_status_t dsc_bwd_lowrank(const void *x, const void *z, const void *U, const void *dy, void *dx,
                             float *dz, float *dU, void *workspace, size_t workspace_bytes, int B,
                             int T, int D, int G, int W, int R, dsc_dtype_t dt,
                             dsc_stream_t stream) {
    const char *fn = "dsc_bwd_lowrank";
    const Dims d{B, T, D, G, W, R};
    dsc_status_t st = check_dims(fn, d, dt);
    if (st != DSC_OK) return st;
    const void *p[] = {x, z, U, dy, dx, dz, dU};
    const char *n[] = {"x", "z", "U", "dy", "dx", "dz", "dU"};
    if ((st = check_ptrs(fn, p, n, 7)) != DSC_OK) return st;
    const bool bf16 = dt == DSC_BF16;
    const size_t need = lowrank_ws(d, bf16);
    if (need) {
        if (workspace_bytes < need)
            return fail(DSC_ERR_UNSUPPORTED, "%s: workspace of %zu bytes is below the %zu required", fn,
                        workspace_bytes, need);
        const void *wp[] = {workspace};
        const char *wn[] = {"workspace"};
        if ((st = check_ptrs(fn, wp, wn, 1)) != DSC_OK) return st;
    }
    if (dsc::tc_lowrank_bwd_supported(B, T, D, G, W, R, bf16))
        return check_launch(fn, dsc::launch_tc_lowrank_bwd(x, z, U, dy, dx, dz, dU, workspace, B, T, D,
                                                           G, W, R, (cudaStream_t)stream));
    dsc::launch_lowrank_bwd_simt(x, z, U, dy, dx, dz, dU, workspace, B, T, D, G, W, R, bf16,
                                 (cudaStream_t)stream);
    return check_launch(fn);
}

DSC_API dsc_status_t dsc_bwd(const void *x, const void *w, const void *dy, void *dx, float *dw, int B, int T,
                     int D, int G, int W, dsc_dtype_t dt, dsc_stream_t stream) {
    const char *fn = "dsc_bwd";
    dsc_status_t st = check_dims(fn, Dims{B, T, D, G, W, -1}, dt);
    if (st != DSC_OK) return st;
    const void *p[] = {x, w, dy, dx, dw};
    const char *n[] = {"x", "w", "dy", "dx", "dw"};
    if ((st = check_ptrs(fn, p, n, 5)) != DSC_OK) return st;
    const bool bf16 = dt == DSC_BF16;
    if (!dsc::launch_dyn_bwd(x, w, dy, dx, dw, B, T, D, G, W, bf16, (cudaStream_t)stream)) {
        dsc::launch_conv_dx(w, false, dy, dx, B, T, D, G, W, bf16, false, (cudaStream_t)stream);
        dsc::launch_dyn_dw(x, dy, dw, B, T, D, G, W, bf16, (cudaStream_t)stream);
    }
    return check_launch(fn);
}

DSC_API dsc_status_t dsc_static_fwd(const void *x, const void *w, void *y, int B, int T, int D, int W,
                            dsc_dtype_t dt, dsc_stream_t stream) {
    const char *fn = "dsc_static_fwd";
    dsc_status_t st = check_dims(fn, Dims{B, T, D, 1, W, -1}, dt);
    if (st != DSC_OK) return st;
    const void *p[] = {x, w, y};
    const char *n[] = {"x", "w", "y"};
    if ((st = check_ptrs(fn, p, n, 3)) != DSC_OK) return st;
    dsc::launch_conv_fwd(x, w, y, B, T, D, 1, W, dt == DSC_BF16, true, (cudaStream_t)stream);
    return check_launch(fn);
}

DSC_API size_t dsc_static_bwd_workspace_bytes(int B, int T, int D, int W, dsc_dtype_t dt) {
    if (check_dims("dsc_static_bwd_workspace_bytes", Dims{B, T, D, 1, W, -1}, dt) != DSC_OK) return 0;
    return (size_t)dsc::static_dw_partials(B, T) * D * W * sizeof(float);
}

DSC_API dsc_status_t dsc_static_bwd(const void *x, const void *w, const void *dy, void *dx, float *dw,
                            void *workspace, size_t workspace_bytes, int B, int T, int D, int W,
                            dsc_dtype_t dt, dsc_stream_t stream) {
    const char *fn = "dsc_static_bwd";
    dsc_status_t st = check_dims(fn, Dims{B, T, D, 1, W, -1}, dt);
    if (st != DSC_OK) return st;
    const void *p[] = {x, w, dy, dx, dw, workspace};
    const char *n[] = {"x", "w", "dy", "dx", "dw", "workspace"};
    if ((st = check_ptrs(fn, p, n, 6)) != DSC_OK) return st;
    const size_t need = dsc_static_bwd_workspace_bytes(B, T, D, W, dt);
    if (workspace_bytes < need)
        return fail(DSC_ERR_UNSUPPORTED, "%s: workspace of %zu bytes is below the %zu required", fn,
                    workspace_bytes, need);
    const bool bf16 = dt == DSC_BF16;
    dsc::launch_static_bwd(x, w, dy, dx, (float *)workspace, dw, B, T, D, W, bf16, (cudaStream_t)stream);
    return check_launch(fn);
}

DSC_API dsc_status_t dsc_decode_step(const void *x_t, const void *w_t, void *state, void *y_t, int B, int D,
                                     int G, int W, dsc_dtype_t dt, dsc_stream_t stream) {
    const char *fn = "dsc_decode_step";
    dsc_status_t st = check_dims(fn, Dims{B, 1, D, G, W, -1}, dt);
    if (st != DSC_OK) return st;
    const void *p[] = {x_t, w_t, y_t};
    const char *n[] = {"x_t", "w_t", "y_t"};
    if ((st = check_ptrs(fn, p, n, 3)) != DSC_OK) return st;
    if (W > 1) {
        const void *sp[] = {state};
        const char *sn[] = {"state"};
        if ((st = check_ptrs(fn, sp, sn, 1)) != DSC_OK) return st;
    }
    return check_launch(fn, dsc::launch_decode(x_t, w_t, state, y_t, B, D, G, W, dt == DSC_BF16,
                                               (cudaStream_t)stream));
}

DSC_API dsc_status_t dsc_decode_step_lowrank(const void *x_t, const void *z_t, const void *U, void *state,
                                             void *y_t, int B, int D, int G, int W, int R, dsc_dtype_t dt,
                                             dsc_stream_t stream) {
    const char *fn = "dsc_decode_step_lowrank";
    dsc_status_t st = check_dims(fn, Dims{B, 1, D, G, W, R}, dt);
    if (st != DSC_OK) return st;
    const void *p[] = {x_t, z_t, U, y_t};
    const char *n[] = {"x_t", "z_t", "U", "y_t"};
    if ((st = check_ptrs(fn, p, n, 4)) != DSC_OK) return st;
    if (W > 1) {
        const void *sp[] = {state};
        const char *sn[] = {"state"};
        if ((st = check_ptrs(fn, sp, sn, 1)) != DSC_OK) return st;
    }
    // tensor cores for w = z U when the batch fills enough of a 128-row tile, else CUDA cores
    if (B >= DSC_DECODE_TC_MIN_B && dsc::tc_decode_lowrank_supported(B, D, G, W, R, dt == DSC_BF16))
        return check_launch(fn, dsc::launch_tc_decode_lowrank(x_t, z_t, U, state, y_t, B, D, G, W, R,
                                                              (cudaStream_t)stream));
    if (!dsc::decode_supported(D, G, W, R))
        return fail(DSC_ERR_UNSUPPORTED, "%s: R=%d with W=%d needs more shared memory than a block has", fn, R, W);
    return check_launch(fn, dsc::launch_decode_lowrank(x_t, z_t, U, state, y_t, B, D, G, W, R, dt == DSC_BF16,
                                                       (cudaStream_t)stream));
}

namespace {
dsc_status_t check_rope(const char *fn, const float *cs, int D, int dh, int n_rot, bool on_tc) {
    if (dh < 16 || dh % 16 || n_rot < 0 || n_rot > D || (n_rot % dh))
        return fail(DSC_ERR_INVALID_ARG, "%s: dh=%d must be a positive multiple of 16 and n_rot=%d a multiple of dh "
                    "within [0, D=%d]", fn, dh, n_rot, D);
    if (n_rot > 0) {
        const void *p[] = {cs};
        const char *n[] = {"cs"};
        dsc_status_t st = check_ptrs(fn, p, n, 1);
        if (st != DSC_OK) return st;
    }
    if (!on_tc)
        return fail(DSC_ERR_UNSUPPORTED, "%s: these sizes are not on the tensor-core path (dsc_lowrank_path)", fn);
    return DSC_OK;
}
}  // namespace

DSC_API dsc_status_t dsc_fwd_lowrank_rope(const void *x, const void *z, const void *U, const float *cs, void *y,
                                          int B, int T, int D, int G, int W, int R, int dh, int n_rot,
                                          dsc_dtype_t dt, dsc_stream_t stream) {
    const char *fn = "dsc_fwd_lowrank_rope";
    dsc_status_t st = check_dims(fn, Dims{B, T, D, G, W, R}, dt);
    if (st != DSC_OK) return st;
    const void *p[] = {x, z, U, y};
    const char *n[] = {"x", "z", "U", "y"};
    if ((st = check_ptrs(fn, p, n, 4)) != DSC_OK) return st;
    const bool bf16 = dt == DSC_BF16;
    if ((st = check_rope(fn, cs, D, dh, n_rot, dsc::tc_lowrank_fwd_supported(B, T, D, G, W, R, bf16))) != DSC_OK)
        return st;
    return check_launch(fn, dsc::launch_tc_lowrank_fwd(x, z, U, y, B, T, D, G, W, R, (cudaStream_t)stream,
                                                       n_rot > 0 ? cs : nullptr, dh, n_rot));
}

DSC_API dsc_status_t dsc_bwd_lowrank_rope(const void *x, const void *z, const void *U, const float *cs,
                                          const void *dy_rot, void *dx, float *dz, float *dU, void *workspace,
                                          size_t workspace_bytes, int B, int T, int D, int G, int W, int R, int dh,
                                          int n_rot, dsc_dtype_t dt, dsc_stream_t stream) {
    const char *fn = "dsc_bwd_lowrank_rope";
    const Dims d{B, T, D, G, W, R};
    dsc_status_t st = check_dims(fn, d, dt);
    if (st != DSC_OK) return st;
    const void *p[] = {x, z, U, dy_rot, dx, dz, dU};
    const char *n[] = {"x", "z", "U", "dy_rot", "dx", "dz", "dU"};
    if ((st = check_ptrs(fn, p, n, 7)) != DSC_OK) return st;
    const bool bf16 = dt == DSC_BF16;
    if ((st = check_rope(fn, cs, D, dh, n_rot, dsc::tc_lowrank_bwd_supported(B, T, D, G, W, R, bf16))) != DSC_OK)
        return st;
    const size_t need = lowrank_ws(d, bf16);
    if (workspace_bytes < need)
        return fail(DSC_ERR_UNSUPPORTED, "%s: workspace of %zu bytes is below the %zu required", fn, workspace_bytes,
                    need);
    const void *wp[] = {workspace};
    const char *wn[] = {"workspace"};
    if ((st = check_ptrs(fn, wp, wn, 1)) != DSC_OK) return st;
    return check_launch(fn, dsc::launch_tc_lowrank_bwd(x, z, U, dy_rot, dx, dz, dU, workspace, B, T, D, G, W, R,
                                                       (cudaStream_t)stream, n_rot > 0 ? cs : nullptr, dh, n_rot));
}

DSC_API dsc_status_t dsc_fwd_lowrank_halo(const void *x, const void *z, const void *U, const void *x_prev,
                                          void *y, int B, int T, int D, int G, int W, int R, dsc_dtype_t dt,
                                          dsc_stream_t stream) {
    const char *fn = "dsc_fwd_lowrank_halo";
    dsc_status_t st = check_dims(fn, Dims{B, T, D, G, W, R}, dt);
    if (st != DSC_OK) return st;
    const void *p[] = {x, z, U, y};
    const char *n[] = {"x", "z", "U", "y"};
    if ((st = check_ptrs(fn, p, n, 4)) != DSC_OK) return st;
    if (x_prev && W > 1) {
        const void *hp[] = {x_prev};
        const char *hn[] = {"x_prev"};
        if ((st = check_ptrs(fn, hp, hn, 1)) != DSC_OK) return st;
    }
    return check_launch(fn, dsc::launch_halo_fwd_lowrank(x, z, U, x_prev, y, B, T, D, G, W, R, dt == DSC_BF16,
                                                         (cudaStream_t)stream));
}

DSC_API dsc_status_t dsc_bwd_lowrank_halo(const void *x_prev, const void *z, const void *U, const void *dy,
                                          const void *dy_next, const void *z_next, void *dx, float *dz,
                                          float *dU, int B, int T, int D, int G, int W, int R, dsc_dtype_t dt,
                                          dsc_stream_t stream) {
    const char *fn = "dsc_bwd_lowrank_halo";
    dsc_status_t st = check_dims(fn, Dims{B, T, D, G, W, R}, dt);
    if (st != DSC_OK) return st;
    const void *p[] = {z, U, dy, dx, dz, dU};
    const char *n[] = {"z", "U", "dy", "dx", "dz", "dU"};
    if ((st = check_ptrs(fn, p, n, 6)) != DSC_OK) return st;
    if ((dy_next == nullptr) != (z_next == nullptr))
        return fail(DSC_ERR_INVALID_ARG, "%s: dy_next and z_next must both be given or both be NULL", fn);
    if (W > 1) {
        const void *hp[] = {x_prev, dy_next, z_next};
        const char *hn[] = {"x_prev", "dy_next", "z_next"};
        for (int i = 0; i < 3; ++i)
            if (hp[i] && (st = check_ptrs(fn, hp + i, hn + i, 1)) != DSC_OK) return st;
    }
    return check_launch(fn, dsc::launch_halo_bwd_lowrank(x_prev, z, U, dy, dy_next, z_next, dx, dz, dU, B, T, D, G,
                                                         W, R, dt == DSC_BF16, (cudaStream_t)stream));
}

DSC_API int dsc_lowrank_path(int B, int T, int D, int G, int W, int R, dsc_dtype_t dt) {
    if (check_dims("dsc_lowrank_path", Dims{B, T, D, G, W, R}, dt) != DSC_OK) return -1;
    const bool bf16 = dt == DSC_BF16;
    return (dsc::tc_lowrank_fwd_supported(B, T, D, G, W, R, bf16) ? 1 : 0) |
           (dsc::tc_lowrank_bwd_supported(B, T, D, G, W, R, bf16) ? 2 : 0);
}

DSC_API unsigned dsc_device_fault(int reset) { return dsc::read_device_fault(reset != 0); }

DSC_API void dsc_test_arm_wait_timeout(unsigned wait_limit_us) {
    dsc::g_test_wait_ns = (unsigned long long)(wait_limit_us ? wait_limit_us : 1) * 1000ull;
}

DSC_API const char *dsc_status_string(dsc_status_t s) {
    switch (s) {
        case DSC_OK: return "DSC_OK";
        case DSC_ERR_INVALID_ARG: return "DSC_ERR_INVALID_ARG: invalid argument";
        case DSC_ERR_UNSUPPORTED: return "DSC_ERR_UNSUPPORTED: unsupported size, alignment or workspace";
        case DSC_ERR_CUDA: return "DSC_ERR_CUDA: CUDA launch error";
    }
    return "unknown dsc status";
}

DSC_API const char *dsc_last_error(void) { return g_err; }

}  // extern "C"
