// Sequence-sharded low-rank dynamic short convolution: the (W-1)-row halo fix-ups.
//
// When a sequence of length P*T is split into P shards of T tokens on P ranks, each
// rank runs dsc_fwd_lowrank / dsc_bwd_lowrank on its shard as if the shard were a whole
// sequence (inputs before its first token read as zero, and no token follows its
// last).  The causal window of "Convolucoes Curtas Dinamicas Melhoram Transformers"
// (Metodologia: Mecanismo, y_t = x_t + sum_{k<W} w(t)_k x_{t-k}) reaches only W-1
// tokens back, so the shard results differ from the unsharded ones in W-1 rows only:
//   forward:  y[t] for t < W-1 reads x of the previous shard's last W-1 rows (x_prev);
//   backward: dx[t] for t >= T-(W-1) reads dy and w = zU of the next shard's first W-1
//             rows (dy_next, z_next); dw[t, g, k] for t < W-1 and k > t reads x_prev,
//             which adds to dz of those rows and to dU.
// These kernels apply exactly those terms after the shard's own call, on the same
// stream: the forward rows and the backward dx rows are recomputed whole (one rounding,
// as in the unsharded kernels); dz and dU receive the missing sums in fp32.  They are
// small (W-1 rows per sequence) CUDA-core kernels with fixed summation orders.
#include "common.cuh"
#include "internal.h"

namespace dsc {
namespace {

constexpr int kHaloThreads = 256;

// w[g, k] of one token: sum_r z[r] U[r, g*W + k], fp32.
template <typename T>
__device__ __forceinline__ float filter_at(const float *zs, const T *__restrict__ U, int R, int N, int col) {
    float w = 0.f;
    for (int r = 0; r < R; ++r) w = fmaf(zs[r], to_f(U[(size_t)r * N + col]), w);
    return w;
}

// y rows t < min(W-1, T) of each sequence, with x[t-k] for t-k < 0 taken from x_prev
// (row W-1+(t-k) of x_prev[b], oldest first).  One block per (b, t), threads over channels.
template <typename T>
__global__ void __launch_bounds__(kHaloThreads)
k_halo_fwd(const T *__restrict__ x, const T *__restrict__ z, const T *__restrict__ U,
           const T *__restrict__ xprev, T *__restrict__ y, int B, int Tn, int D, int G, int W, int R) {
    extern __shared__ float zs[];                 // z[b, t, :]
    const int rows = min(W - 1, Tn);
    const int N = (D / G) * W;
    for (long long blk = blockIdx.x; blk < (long long)B * rows; blk += gridDim.x) {
        const int b = (int)(blk / rows), t = (int)(blk - (long long)b * rows);
        __syncthreads();
        for (int r = threadIdx.x; r < R; r += blockDim.x) zs[r] = to_f(z[((size_t)b * Tn + t) * R + r]);
        __syncthreads();
        for (int c = threadIdx.x; c < D; c += blockDim.x) {
            const int g = c / G;
            float acc = to_f(x[((size_t)b * Tn + t) * D + c]);
            for (int k = 0; k < W; ++k) {
                const int s = t - k;
                const float xv = s >= 0 ? to_f(x[((size_t)b * Tn + s) * D + c])
                                        : to_f(xprev[((size_t)b * (W - 1) + (W - 1 + s)) * D + c]);
                acc = fmaf(filter_at(zs, U, R, N, g * W + k), xv, acc);
            }
            y[((size_t)b * Tn + t) * D + c] = from_f<T>(acc);
        }
    }
}

// dx rows t >= T-(W-1) of each sequence: dx[t] = dy[t] + sum_k w[t+k, g, k] dy[t+k], with
// rows t+k >= T taken from dy_next / z_next (row t+k-T).  One block per (b, row).
template <typename T>
__global__ void __launch_bounds__(kHaloThreads)
k_halo_dx(const T *__restrict__ z, const T *__restrict__ U, const T *__restrict__ dy,
          const T *__restrict__ dy_next, const T *__restrict__ z_next, T *__restrict__ dx, int B, int Tn,
          int D, int G, int W, int R) {
    extern __shared__ float zs[];                 // z of rows t .. t+W-1, [W][R]
    const int rows = min(W - 1, Tn);
    const int N = (D / G) * W;
    for (long long blk = blockIdx.x; blk < (long long)B * rows; blk += gridDim.x) {
        const int b = (int)(blk / rows);
        const int t = Tn - rows + (int)(blk - (long long)b * rows);
        __syncthreads();
        for (int e = threadIdx.x; e < W * R; e += blockDim.x) {
            const int k = e / R, r = e - k * R, tt = t + k;
            zs[e] = tt < Tn ? to_f(z[((size_t)b * Tn + tt) * R + r])
                            : to_f(z_next[((size_t)b * (W - 1) + (tt - Tn)) * R + r]);
        }
        __syncthreads();
        for (int c = threadIdx.x; c < D; c += blockDim.x) {
            const int g = c / G;
            float acc = to_f(dy[((size_t)b * Tn + t) * D + c]);
            for (int k = 0; k < W; ++k) {
                const int tt = t + k;
                const float d = tt < Tn ? to_f(dy[((size_t)b * Tn + tt) * D + c])
                                        : to_f(dy_next[((size_t)b * (W - 1) + (tt - Tn)) * D + c]);
                acc = fmaf(filter_at(zs + k * R, U, R, N, g * W + k), d, acc);
            }
            dx[((size_t)b * Tn + t) * D + c] = from_f<T>(acc);
        }
    }
}

// The filter gradient terms the shard's call left out: for t < min(W-1, T) and k > t,
//   ddw[b, t, g, k] = sum_{c in g} dy[b, t, c] x_prev[b, W-1+t-k, c].
template <typename T>
__device__ __forceinline__ float halo_dw(const T *__restrict__ dy, const T *__restrict__ xprev, int b, int t,
                                         int g, int k, int Tn, int D, int G, int W) {
    const T *d = dy + ((size_t)b * Tn + t) * D + (size_t)g * G;
    const T *xp = xprev + ((size_t)b * (W - 1) + (W - 1 + t - k)) * D + (size_t)g * G;
    float s = 0.f;
    for (int e = 0; e < G; ++e) s = fmaf(to_f(d[e]), to_f(xp[e]), s);
    return s;
}

// dz[b, t, r] += sum_{g, k > t} ddw[b, t, g, k] U[r, g*W + k].  One block per (b, t, group
// of 8 r); the threads stride over the columns and a fixed-order shared-memory tree sums them.
constexpr int kRC = 8;
template <typename T>
__global__ void __launch_bounds__(kHaloThreads)
k_halo_dz(const T *__restrict__ xprev, const T *__restrict__ U, const T *__restrict__ dy, float *__restrict__ dz,
          int B, int Tn, int D, int G, int W, int R) {
    __shared__ float red[kRC][kHaloThreads];
    const int rows = min(W - 1, Tn);
    const int nrc = cdiv(R, kRC);
    const int NG = D / G, N = NG * W;
    for (long long blk = blockIdx.x; blk < (long long)B * rows * nrc; blk += gridDim.x) {
        const int rc = (int)(blk % nrc);
        const long long bt = blk / nrc;
        const int b = (int)(bt / rows), t = (int)(bt - (long long)b * rows);
        const int r0 = rc * kRC;
        float acc[kRC];
#pragma unroll
        for (int i = 0; i < kRC; ++i) acc[i] = 0.f;
        const int kn = W - 1 - t;                 // taps k = t+1 .. W-1
        for (int e = threadIdx.x; e < NG * kn; e += blockDim.x) {
            const int g = e / kn, k = t + 1 + (e - g * kn);
            const float v = halo_dw(dy, xprev, b, t, g, k, Tn, D, G, W);
#pragma unroll
            for (int i = 0; i < kRC; ++i)
                if (r0 + i < R) acc[i] = fmaf(v, to_f(U[(size_t)(r0 + i) * N + g * W + k]), acc[i]);
        }
        __syncthreads();
#pragma unroll
        for (int i = 0; i < kRC; ++i) red[i][threadIdx.x] = acc[i];
        __syncthreads();
        for (int h = kHaloThreads / 2; h > 0; h >>= 1) {
            if ((int)threadIdx.x < h)
#pragma unroll
                for (int i = 0; i < kRC; ++i) red[i][threadIdx.x] += red[i][threadIdx.x + h];
            __syncthreads();
        }
        if ((int)threadIdx.x < kRC && r0 + (int)threadIdx.x < R)
            dz[((size_t)b * Tn + t) * R + r0 + threadIdx.x] += red[threadIdx.x][0];
    }
}

// dU[r, g*W + k] += sum_{b, t < min(W-1, T), t < k} z[b, t, r] ddw[b, t, g, k].  One block per
// 32 columns: the ddw of 64 (b, t) pairs at a time go to shared memory, then thread (column
// jl, row group rg) accumulates rows r = rg, rg+8, ... over the pairs in order.
constexpr int kPairs = 64;
constexpr int kMaxRPerThread = 32;                // R <= 256
template <typename T>
__global__ void __launch_bounds__(kHaloThreads)
k_halo_du(const T *__restrict__ xprev, const T *__restrict__ z, const T *__restrict__ dy, float *__restrict__ dU,
          int B, int Tn, int D, int G, int W, int R) {
    __shared__ float dws[kPairs][32];
    const int rows = min(W - 1, Tn);
    const int NG = D / G, N = NG * W;
    const long long npairs = (long long)B * rows;
    const int jl = threadIdx.x & 31, rg = threadIdx.x >> 5;
    for (int j0 = blockIdx.x * 32; j0 < N; j0 += gridDim.x * 32) {
        float acc[kMaxRPerThread];
#pragma unroll
        for (int i = 0; i < kMaxRPerThread; ++i) acc[i] = 0.f;
        for (long long p0 = 0; p0 < npairs; p0 += kPairs) {
            __syncthreads();
            for (int e = threadIdx.x; e < kPairs * 32; e += blockDim.x) {
                const int pl = e >> 5, jj = e & 31;
                const long long pr = p0 + pl;
                const int j = j0 + jj;
                float v = 0.f;
                if (pr < npairs && j < N) {
                    const int b = (int)(pr / rows), t = (int)(pr - (long long)b * rows);
                    const int g = j / W, k = j - g * W;
                    if (k > t) v = halo_dw(dy, xprev, b, t, g, k, Tn, D, G, W);
                }
                dws[pl][jj] = v;
            }
            __syncthreads();
            const int np = (int)min((long long)kPairs, npairs - p0);
            for (int pl = 0; pl < np; ++pl) {
                const long long pr = p0 + pl;
                const int b = (int)(pr / rows), t = (int)(pr - (long long)b * rows);
                const T *zr = z + ((size_t)b * Tn + t) * R;
                const float v = dws[pl][jl];
#pragma unroll
                for (int i = 0; i < kMaxRPerThread; ++i) {
                    const int r = rg + 8 * i;
                    if (r < R) acc[i] = fmaf(to_f(zr[r]), v, acc[i]);
                }
            }
        }
        const int j = j0 + jl;
        if (j < N) {
#pragma unroll
            for (int i = 0; i < kMaxRPerThread; ++i) {
                const int r = rg + 8 * i;
                if (r < R) dU[(size_t)r * N + j] += acc[i];
            }
        }
    }
}

// Grid of a halo kernel: one block per work item, at most 64 per SM (the kernels stride).
int halo_grid(long long blocks) { return (int)std::min<long long>(std::max<long long>(blocks, 1), 148ll * 64); }

template <typename T>
cudaError_t halo_fwd_t(const void *x, const void *z, const void *U, const void *xprev, void *y, int B, int Tn,
                       int D, int G, int W, int R, cudaStream_t s) {
    if (W == 1 || !xprev) return cudaSuccess;
    const long long blocks = (long long)B * std::min(W - 1, Tn);
    k_halo_fwd<T><<<halo_grid(blocks), kHaloThreads, R * sizeof(float), s>>>(
        (const T *)x, (const T *)z, (const T *)U, (const T *)xprev, (T *)y, B, Tn, D, G, W, R);
    return cudaGetLastError();
}

template <typename T>
cudaError_t halo_bwd_t(const void *xprev, const void *z, const void *U, const void *dy, const void *dy_next,
                       const void *z_next, void *dx, float *dz, float *dU, int B, int Tn, int D, int G, int W,
                       int R, cudaStream_t s) {
    if (W == 1) return cudaSuccess;
    const int rows = std::min(W - 1, Tn);
    if (dy_next) {
        k_halo_dx<T><<<halo_grid((long long)B * rows), kHaloThreads, W * R * sizeof(float), s>>>(
            (const T *)z, (const T *)U, (const T *)dy, (const T *)dy_next, (const T *)z_next, (T *)dx, B, Tn, D, G, W, R);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    if (xprev) {
        k_halo_dz<T><<<halo_grid((long long)B * rows * cdiv(R, kRC)), kHaloThreads, 0, s>>>(
            (const T *)xprev, (const T *)U, (const T *)dy, dz, B, Tn, D, G, W, R);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        const int N = (D / G) * W;
        k_halo_du<T><<<halo_grid(cdiv(N, 32)), kHaloThreads, 0, s>>>((const T *)xprev, (const T *)z, (const T *)dy,
                                                                      dU, B, Tn, D, G, W, R);
        return cudaGetLastError();
    }
    return cudaSuccess;
}

}  // namespace

cudaError_t launch_halo_fwd_lowrank(const void *x, const void *z, const void *U, const void *x_prev, void *y,
                                    int B, int T, int D, int G, int W, int R, bool is_bf16, cudaStream_t s) {
    return is_bf16 ? halo_fwd_t<bf16>(x, z, U, x_prev, y, B, T, D, G, W, R, s)
                : halo_fwd_t<float>(x, z, U, x_prev, y, B, T, D, G, W, R, s);
}

cudaError_t launch_halo_bwd_lowrank(const void *x_prev, const void *z, const void *U, const void *dy,
                                    const void *dy_next, const void *z_next, void *dx, float *dz, float *dU,
                                    int B, int T, int D, int G, int W, int R, bool is_bf16, cudaStream_t s) {
    return is_bf16 ? halo_bwd_t<bf16>(x_prev, z, U, dy, dy_next, z_next, dx, dz, dU, B, T, D, G, W, R, s)
                : halo_bwd_t<float>(x_prev, z, U, dy, dy_next, z_next, dx, dz, dU, B, T, D, G, W, R, s);
}

}  // namespace dsc
