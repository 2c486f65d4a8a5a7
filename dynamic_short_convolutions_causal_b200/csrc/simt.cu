// CUDA-core kernels: the explicit-filter backward (dx and the per-token filter
// gradient), and the general-shape low-rank path used where the tensor-core kernels
// do not apply (fp32, or R / G / W outside the tensor-core shapes).  The forward
// kernels and the static backward are in stream.cu.
//
// The operation is the causal dynamic short convolution of "Convolucoes Curtas
// Dinamicas Melhoram Transformers" (Metodologia > Convolucoes Curtas Dinamicas):
//   y_t[c] = x_t[c] + sum_{k<W} f_t[c,k] x_{t-k}[c],   x_{t'} = 0 for t' < 0,
// and its chain-rule backward.
//
// Streaming layout: one thread owns one 16-byte vector of channels (8 bf16 or 4 fp32)
// and walks a chunk of tokens of one sequence, keeping the W-1 previous rows of x in
// registers, so x and y each cross HBM once (the W-1 halo rows at a chunk start are
// re-read, mostly from L2).
#include "common.cuh"
#include "internal.h"

namespace dsc {

// Filter taps for the thread's V channels at token row `bt` (flattened b*T+t).
//   STATIC:  ws[c,k]                  (loaded once by the caller)
//   G == 1:  w[bt, c, k] contiguous   (V*W elements, 16-byte vectors)
//   G % V == 0: one group for all V channels (W elements)
//   else:    per channel
template <typename T, typename TW, int W>
__device__ __forceinline__ void load_taps(const TW *__restrict__ w, size_t bt, int c0, int D,
                                          int G, float (&f)[W][Vec<T>::N]) {
    constexpr int V = Vec<T>::N;
    const int NG = D / G;
    if (G == 1 && sizeof(TW) == sizeof(T)) {
        // V*W contiguous elements; (bt*D + c0)*W*sizeof(TW) is a multiple of 16.
        const TW *p = w + (bt * (size_t)D + c0) * W;
        float tmp[V * W];
#pragma unroll
        for (int q = 0; q < W; ++q) {
            float v[V];
            Vec<T>::load(reinterpret_cast<const T *>(p) + q * V, v);
#pragma unroll
            for (int e = 0; e < V; ++e) tmp[q * V + e] = v[e];
        }
#pragma unroll
        for (int i = 0; i < V; ++i)
#pragma unroll
            for (int k = 0; k < W; ++k) f[k][i] = tmp[i * W + k];
    } else if (G % V == 0) {
        const TW *p = w + (bt * NG + c0 / G) * W;
        float t[W];
#pragma unroll
        for (int k = 0; k < W; ++k) t[k] = to_f(p[k]);
#pragma unroll
        for (int i = 0; i < V; ++i)
#pragma unroll
            for (int k = 0; k < W; ++k) f[k][i] = t[k];
    } else {
#pragma unroll
        for (int i = 0; i < V; ++i) {
            const TW *p = w + (bt * NG + (c0 + i) / G) * W;
#pragma unroll
            for (int k = 0; k < W; ++k) f[k][i] = to_f(p[k]);
        }
    }
}

// ------------------------------------------------------------------ dx (scatter form)
// Walks t upward through [t0, t1 + W - 1): at token t the products w_t[.,k] * dy_t are
// added into the open rows t-k; row t-W+1 is complete after token t.  Rows outside
// [t0, t1) belong to neighbouring chunks and are not stored.
//   STATIC: taps ws[c,k]; otherwise per-token taps w (type TW, G-tied).
template <typename T, typename TW, int W, bool STATIC>
__global__ void __launch_bounds__(128)
k_conv_bwd_dx(const TW *__restrict__ w, const T *__restrict__ dy, T *__restrict__ dx,
              int B, int T_, int D, int G, int chunk) {
    constexpr int V = Vec<T>::N;
    const int v = blockIdx.x * blockDim.x + threadIdx.x;
    if (v >= D / V) return;
    const int nchunks = cdiv(T_, chunk);
    const int b = blockIdx.y / nchunks;
    const int t0 = (blockIdx.y % nchunks) * chunk;
    const int t1 = min(t0 + chunk, T_);
    const int tend = min(t1 + W - 1, T_);
    const int c0 = v * V;
    const size_t row0 = (size_t)b * T_;

    float acc[W][V];   // acc[k] = partial dx of row t-k
#pragma unroll
    for (int k = 0; k < W; ++k)
#pragma unroll
        for (int i = 0; i < V; ++i) acc[k][i] = 0.f;
    float f[W][V];
    if (STATIC) {
#pragma unroll
        for (int i = 0; i < V; ++i)
#pragma unroll
            for (int k = 0; k < W; ++k) f[k][i] = to_f(w[(size_t)(c0 + i) * W + k]);
    }
    for (int t = t0; t < tend; ++t) {
        const size_t bt = row0 + t;
        float g[V];
        Vec<T>::load(dy + bt * D + c0, g);
        if (!STATIC) load_taps<T, TW, W>(w, bt, c0, D, G, f);
#pragma unroll
        for (int i = 0; i < V; ++i) acc[0][i] = (t < t1) ? g[i] : 0.f;   // residual
#pragma unroll
        for (int k = 0; k < W; ++k)
#pragma unroll
            for (int i = 0; i < V; ++i) acc[k][i] = fmaf(f[k][i], g[i], acc[k][i]);
        const int done = t - (W - 1);
        if (done >= t0 && done < t1) Vec<T>::store(dx + (row0 + done) * D + c0, acc[W - 1]);
#pragma unroll
        for (int k = W - 1; k >= 1; --k)
#pragma unroll
            for (int i = 0; i < V; ++i) acc[k][i] = acc[k - 1][i];
    }
    // Sequence end: the still-open rows received all their contributions.
    // After the shift, acc[k] holds row (tend - k) for k = 1..W-1.
#pragma unroll
    for (int k = 1; k < W; ++k) {
        const int row = tend - k;
        if (tend == T_ && row >= t0 && row < t1 && row > tend - W)
            Vec<T>::store(dx + (row0 + row) * D + c0, acc[k]);
    }
}

// ------------------------------------------------------------------ explicit dw, rows
// dw[bt,g,k] = sum_{c in g, t-k >= 0} dy[bt,c] x[bt-k,c] with the channels along the
// threads: a thread owns one 16-byte vector (V channels) and walks a chunk of tokens with
// the W rows x[t-k] in registers, so each row of x and dy is read once, coalesced.  Its
// V products per tap are summed in the thread (groups of at most V channels: V/G groups
// per thread) or across the G/V threads of a group by a fixed xor-shuffle tree (G a
// multiple of V, G/V <= 32, a power of two); one thread per group writes the W taps.
template <typename T, int W>
__global__ void __launch_bounds__(256)
k_dyn_dw_rows(const T *__restrict__ x, const T *__restrict__ dy, float *__restrict__ dw,
              int B, int T_, int D, int G, int chunk) {
    constexpr int V = Vec<T>::N;
    const int nv = D / V;
    const int v = blockIdx.x * blockDim.x + threadIdx.x;
    const bool active = v < nv;
    const int nchunks = cdiv(T_, chunk);
    const int b = blockIdx.y / nchunks;
    const int t0 = (blockIdx.y % nchunks) * chunk;
    const int t1 = min(t0 + chunk, T_);
    const int c0 = (active ? v : 0) * V;
    const int NG = D / G;
    const int lanes = G > V ? G / V : 1;        // threads per group
    const size_t row0 = (size_t)b * T_;
    float xw[W][V];                             // xw[k] = x[t-k]
#pragma unroll
    for (int k = 1; k < W; ++k) {
        if (active && t0 - k >= 0) Vec<T>::load(x + (row0 + t0 - k) * D + c0, xw[k]);
        else
#pragma unroll
            for (int i = 0; i < V; ++i) xw[k][i] = 0.f;
    }
    for (int t = t0; t < t1; ++t) {
        float g[V];
        if (active) {
            Vec<T>::load(x + (row0 + t) * D + c0, xw[0]);
            Vec<T>::load(dy + (row0 + t) * D + c0, g);
        } else {
#pragma unroll
            for (int i = 0; i < V; ++i) xw[0][i] = g[i] = 0.f;
        }
        float* out = dw + (row0 + t) * (size_t)NG * W;
        if (G >= V) {
            float s[W];
#pragma unroll
            for (int k = 0; k < W; ++k) {
                float a = 0.f;
#pragma unroll
                for (int i = 0; i < V; ++i) a = fmaf(g[i], xw[k][i], a);
                s[k] = a;
            }
            for (int o = 1; o < lanes; o <<= 1)
#pragma unroll
                for (int k = 0; k < W; ++k) s[k] += __shfl_xor_sync(0xffffffffu, s[k], o);
            if (active && (v % lanes) == 0) {
                float *q = out + (size_t)(c0 / G) * W;
#pragma unroll
                for (int k = 0; k < W; ++k) q[k] = s[k];
            }
        } else {
            // V/G whole groups in the thread
            for (int gl = 0; gl < V / G; ++gl) {
                float s[W];
#pragma unroll
                for (int k = 0; k < W; ++k) s[k] = 0.f;
                for (int e = gl * G; e < (gl + 1) * G; ++e)
#pragma unroll
                    for (int k = 0; k < W; ++k) s[k] = fmaf(g[e], xw[k][e], s[k]);
                if (active) {
                    float *q = out + (size_t)(c0 / G + gl) * W;
#pragma unroll
                    for (int k = 0; k < W; ++k) q[k] = s[k];
                }
            }
        }
#pragma unroll
        for (int k = W - 1; k >= 1; --k)
#pragma unroll
            for (int i = 0; i < V; ++i) xw[k][i] = xw[k - 1][i];
    }
}

// ------------------------------------------------------------------ explicit dw
// dw[bt,g,k] = sum_{c in g, t-k >= 0} dy[bt,c] x[bt-k,c]; one thread per (bt, g).
template <typename T>
__global__ void k_dyn_dw(const T *__restrict__ x, const T *__restrict__ dy, float *__restrict__ dw,
                         int B, int T_, int D, int G, int W) {
    const int NG = D / G;
    const size_t n = (size_t)B * T_ * NG;
    for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < n;
         e += (size_t)gridDim.x * blockDim.x) {
        const size_t bt = e / NG;
        const int g = (int)(e % NG);
        const int t = (int)(bt % T_);
        for (int k = 0; k < W; ++k) {
            float s = 0.f;
            if (t - k >= 0) {
                const T *pg = dy + bt * D + (size_t)g * G;
                const T *px = x + (bt - k) * D + (size_t)g * G;
                for (int c = 0; c < G; ++c) s = fmaf(to_f(pg[c]), to_f(px[c]), s);
            }
            dw[e * W + k] = s;
        }
    }
}

// ------------------------------------------------------------------ low-rank, CUDA cores
// Fused forward for general shapes.  Block = TT tokens of one sequence x 64 channels.
// Phase 1 forms the filter tile wt[t][j] = sum_r z[t,r] U[r, jbase + j] in shared memory
// (fp32), phase 2 applies the causal convolution with the residual.
constexpr int kLrTT = 16;
constexpr int kLrCS = 64;
constexpr int kLrMaxCols = (kLrCS + 2) * 8;   // groups touched by 64 channels, W <= 8

template <typename T>
__global__ void __launch_bounds__(256)
k_lowrank_fwd_simt(const T *__restrict__ x, const T *__restrict__ z, const T *__restrict__ U,
                   T *__restrict__ y, int B, int T_, int D, int G, int W, int R) {
    __shared__ float wt[kLrTT][kLrMaxCols];
    extern __shared__ float zs[];   // [kLrTT][R]
    const int NG = D / G;
    const int N = NG * W;
    const int c0 = blockIdx.x * kLrCS;
    const int c1 = min(c0 + kLrCS, D);
    const int ntile = cdiv(T_, kLrTT);
    const int b = blockIdx.y / ntile;
    const int t0 = (blockIdx.y % ntile) * kLrTT;
    const int nt = min(kLrTT, T_ - t0);
    const int g_lo = c0 / G, g_hi = (c1 - 1) / G;
    const int ncols = (g_hi - g_lo + 1) * W;
    const size_t row0 = (size_t)b * T_ + t0;

    for (int e = threadIdx.x; e < kLrTT * R; e += blockDim.x) {
        const int t = e / R, r = e % R;
        zs[e] = (t < nt) ? to_f(z[(row0 + t) * R + r]) : 0.f;
    }
    __syncthreads();
    for (int j = threadIdx.x; j < ncols; j += blockDim.x) {
        float acc[kLrTT];
#pragma unroll
        for (int t = 0; t < kLrTT; ++t) acc[t] = 0.f;
        const int col = g_lo * W + j;
        if (col < N) {
            for (int r = 0; r < R; ++r) {
                const float u = to_f(U[(size_t)r * N + col]);
#pragma unroll
                for (int t = 0; t < kLrTT; ++t) acc[t] = fmaf(zs[t * R + r], u, acc[t]);
            }
        }
#pragma unroll
        for (int t = 0; t < kLrTT; ++t) wt[t][j] = acc[t];
    }
    __syncthreads();
    const int width = c1 - c0;
    for (int e = threadIdx.x; e < nt * width; e += blockDim.x) {
        const int t = e / width, c = c0 + e % width;
        const int gt = t0 + t;
        const int jb = (c / G - g_lo) * W;
        const size_t bt = row0 + t;
        float acc = to_f(x[bt * D + c]);
        for (int k = 0; k < W && gt - k >= 0; ++k)
            acc = fmaf(wt[t][jb + k], to_f(x[(bt - k) * D + c]), acc);
        y[bt * D + c] = from_f<T>(acc);
    }
}

// wm[bt, j] = sum_r z[bt, r] U[r, j] in fp32 (materialised filters for the CUDA-core
// backward).  Block = kLrTT tokens x 256 columns.
template <typename T>
__global__ void __launch_bounds__(256)
k_lowrank_weights(const T *__restrict__ z, const T *__restrict__ U, float *__restrict__ wm,
                  int BT, int N, int R) {
    extern __shared__ float zs[];   // [kLrTT][R]
    const int bt0 = blockIdx.y * kLrTT;
    const int nt = min(kLrTT, BT - bt0);
    for (int e = threadIdx.x; e < kLrTT * R; e += blockDim.x) {
        const int t = e / R, r = e % R;
        zs[e] = (t < nt) ? to_f(z[(size_t)(bt0 + t) * R + r]) : 0.f;
    }
    __syncthreads();
    const int j = blockIdx.x * blockDim.x + threadIdx.x;
    if (j >= N) return;
    float acc[kLrTT];
#pragma unroll
    for (int t = 0; t < kLrTT; ++t) acc[t] = 0.f;
    for (int r = 0; r < R; ++r) {
        const float u = to_f(U[(size_t)r * N + j]);
#pragma unroll
        for (int t = 0; t < kLrTT; ++t) acc[t] = fmaf(zs[t * R + r], u, acc[t]);
    }
    for (int t = 0; t < nt; ++t) wm[(size_t)(bt0 + t) * N + j] = acc[t];
}

// dz[bt, r] = sum_j dw[bt, j] U[r, j]; one warp per token, lanes over j.
template <typename T>
__global__ void __launch_bounds__(256)
k_lowrank_dz(const float *__restrict__ dw, const T *__restrict__ U, float *__restrict__ dz,
             int BT, int N, int R) {
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (warp >= BT) return;
    const float *row = dw + (size_t)warp * N;
    for (int r = 0; r < R; ++r) {
        const T *u = U + (size_t)r * N;
        float s = 0.f;
        for (int j = lane; j < N; j += 32) s = fmaf(row[j], to_f(u[j]), s);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (lane == 0) dz[(size_t)warp * R + r] = s;
    }
}

// dU[r, j] = sum_bt z[bt, r] dw[bt, j], summed over bt in order.
template <typename T>
__global__ void __launch_bounds__(256)
k_lowrank_dU(const T *__restrict__ z, const float *__restrict__ dw, float *__restrict__ dU,
             int BT, int N, int R) {
    const int j = blockIdx.x * blockDim.x + threadIdx.x;
    const int r = blockIdx.y;
    if (j >= N) return;
    float s = 0.f;
    for (int bt = 0; bt < BT; ++bt) s = fmaf(to_f(z[(size_t)bt * R + r]), dw[(size_t)bt * N + j], s);
    dU[(size_t)r * N + j] = s;
}

// ------------------------------------------------------------------ launchers
constexpr int kChunk = 32;

template <typename T, typename TW, bool STATIC>
static void launch_dx_T(const void *w, const void *dy, void *dx, int B, int T_, int D, int G, int W,
                        cudaStream_t s) {
    constexpr int V = Vec<T>::N;
    const dim3 block(128);
    const dim3 grid(cdiv(D / V, 128), B * cdiv(T_, kChunk));
    const TW *wp = (const TW *)w;
    const T *gp = (const T *)dy;
    T *op = (T *)dx;
    switch (W) {
#define DSC_CASE(WW) \
    case WW: k_conv_bwd_dx<T, TW, WW, STATIC><<<grid, block, 0, s>>>(wp, gp, op, B, T_, D, G, kChunk); break;
        DSC_CASE(1) DSC_CASE(2) DSC_CASE(3) DSC_CASE(4) DSC_CASE(5) DSC_CASE(6) DSC_CASE(7) DSC_CASE(8)
#undef DSC_CASE
    }
}

void launch_conv_dx(const void *w, bool w_is_f32, const void *dy, void *dx, int B, int T, int D,
                    int G, int W, bool bf16_, bool is_static, cudaStream_t s) {
    if (bf16_) {
        if (is_static) launch_dx_T<bf16, bf16, true>(w, dy, dx, B, T, D, 1, W, s);
        else if (w_is_f32) launch_dx_T<bf16, float, false>(w, dy, dx, B, T, D, G, W, s);
        else launch_dx_T<bf16, bf16, false>(w, dy, dx, B, T, D, G, W, s);
    } else {
        if (is_static) launch_dx_T<float, float, true>(w, dy, dx, B, T, D, 1, W, s);
        else launch_dx_T<float, float, false>(w, dy, dx, B, T, D, G, W, s);
    }
}

template <typename T>
static bool launch_dw_rows(const void *x, const void *dy, float *dw, int B, int T_, int D, int G, int W,
                           cudaStream_t s) {
    constexpr int V = Vec<T>::N;
    const bool ok = (G >= V) ? (G % V == 0 && (G / V) <= 32 && ((G / V) & (G / V - 1)) == 0) : (V % G == 0);
    if (!ok) return false;
    constexpr int kRowChunk = 64;
    const dim3 grid(cdiv(D / V, 256), B * cdiv(T_, kRowChunk));
    const T *xp = (const T *)x;
    const T *gp = (const T *)dy;
    switch (W) {
#define DSC_CASE(WW) \
    case WW: k_dyn_dw_rows<T, WW><<<grid, 256, 0, s>>>(xp, gp, dw, B, T_, D, G, kRowChunk); break;
        DSC_CASE(1) DSC_CASE(2) DSC_CASE(3) DSC_CASE(4) DSC_CASE(5) DSC_CASE(6) DSC_CASE(7) DSC_CASE(8)
#undef DSC_CASE
    }
    return true;
}

void launch_dyn_dw(const void *x, const void *dy, float *dw, int B, int T, int D, int G, int W,
                   bool bf16_, cudaStream_t s) {
    // row-parallel kernel where the groups tile the threads' channel vectors; otherwise
    // one thread per (token, group)
    if (bf16_ ? launch_dw_rows<bf16>(x, dy, dw, B, T, D, G, W, s) : launch_dw_rows<float>(x, dy, dw, B, T, D, G, W, s))
        return;
    const size_t n = (size_t)B * T * (D / G);
    const unsigned grid = (unsigned)std::min<size_t>((n + 255) / 256, 65535u * 8);
    if (bf16_) k_dyn_dw<bf16><<<grid, 256, 0, s>>>((const bf16 *)x, (const bf16 *)dy, dw, B, T, D, G, W);
    else k_dyn_dw<float><<<grid, 256, 0, s>>>((const float *)x, (const float *)dy, dw, B, T, D, G, W);
}

void launch_lowrank_fwd_simt(const void *x, const void *z, const void *U, void *y, int B, int T,
                             int D, int G, int W, int R, bool bf16_, cudaStream_t s) {
    const dim3 grid(cdiv(D, kLrCS), B * cdiv(T, kLrTT));
    const size_t smem = sizeof(float) * kLrTT * R;
    if (bf16_)
        k_lowrank_fwd_simt<bf16><<<grid, 256, smem, s>>>((const bf16 *)x, (const bf16 *)z,
                                                         (const bf16 *)U, (bf16 *)y, B, T, D, G, W, R);
    else
        k_lowrank_fwd_simt<float><<<grid, 256, smem, s>>>((const float *)x, (const float *)z,
                                                          (const float *)U, (float *)y, B, T, D, G, W, R);
}

size_t lowrank_bwd_simt_workspace(int B, int T, int D, int G, int W) {
    const size_t n = (size_t)B * T * (D / G) * W;
    return 2 * n * sizeof(float);
}

void launch_lowrank_bwd_simt(const void *x, const void *z, const void *U, const void *dy, void *dx,
                             float *dz, float *dU, void *ws, int B, int T, int D, int G, int W,
                             int R, bool bf16_, cudaStream_t s) {
    const int BT = B * T;
    const int N = (D / G) * W;
    float *wm = (float *)ws;
    float *dwm = wm + (size_t)BT * N;
    const dim3 gw(cdiv(N, 256), cdiv(BT, kLrTT));
    const size_t smem = sizeof(float) * kLrTT * R;
    if (bf16_) k_lowrank_weights<bf16><<<gw, 256, smem, s>>>((const bf16 *)z, (const bf16 *)U, wm, BT, N, R);
    else k_lowrank_weights<float><<<gw, 256, smem, s>>>((const float *)z, (const float *)U, wm, BT, N, R);
    launch_conv_dx(wm, true, dy, dx, B, T, D, G, W, bf16_, false, s);
    launch_dyn_dw(x, dy, dwm, B, T, D, G, W, bf16_, s);
    const unsigned gz = (unsigned)cdiv(BT, 8);
    const dim3 gU(cdiv(N, 256), R);
    if (bf16_) {
        k_lowrank_dz<bf16><<<gz, 256, 0, s>>>(dwm, (const bf16 *)U, dz, BT, N, R);
        k_lowrank_dU<bf16><<<gU, 256, 0, s>>>((const bf16 *)z, dwm, dU, BT, N, R);
    } else {
        k_lowrank_dz<float><<<gz, 256, 0, s>>>(dwm, (const float *)U, dz, BT, N, R);
        k_lowrank_dU<float><<<gU, 256, 0, s>>>((const float *)z, dwm, dU, BT, N, R);
    }
}

}  // namespace dsc
