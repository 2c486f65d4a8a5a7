// Single-token decode step of the causal dynamic short convolution, for B sequences at
// once, each with a caller-owned rolling window of its W-1 previous inputs.
//
// "Convolucoes Curtas Dinamicas Melhoram Transformers": the Mecanismo formula at one
// position t,
//   y_t[c] = x_t[c] + w_t[g(c),0] x_t[c] + sum_{k=1}^{W-1} w_t[g(c),k] x_{t-k}[c],
// with x_{t-k} read from the window (row W-1-k of state [B, W-1, D], oldest first);
// the window is then shifted by one row and x_t appended, in place.  The page notes
// that inference still needs engineering (Significancia e Alegacoes); this is the
// step a generation loop calls once per token.
//
// Low-rank filters w_t = z_t U are formed per step.  A block owns 32 channels and up
// to 32 sequences: it stages z and the U columns of its channels in shared memory as
// fp32, forms w for its sequences and columns with 4x4 register tiles (16 FMAs per
// two 16-byte shared loads), then applies the convolution, one thread per
// (sequence, 4 channels).  Every call reads U once per block of sequences; for large B
// the step is bound by the FMAs of w (2*R*N per sequence) on the CUDA cores.
#include "common.cuh"
#include "internal.h"

namespace dsc {

namespace {

constexpr int kDcCh = 32;          // channels per block
constexpr int kDcSeq = 32;         // sequences per block
constexpr int kDcThreads = 256;

// Loads 4 consecutive channels (one 8- or 16-byte vector) as floats.
template <typename T>
__device__ __forceinline__ void ld4(const T *p, float (&v)[4]) {
    if constexpr (sizeof(T) == 2) {
        const uint2 u = *reinterpret_cast<const uint2 *>(p);
        v[0] = bf16_lo(u.x); v[1] = bf16_hi(u.x); v[2] = bf16_lo(u.y); v[3] = bf16_hi(u.y);
    } else {
        const float4 u = *reinterpret_cast<const float4 *>(p);
        v[0] = u.x; v[1] = u.y; v[2] = u.z; v[3] = u.w;
    }
}
template <typename T>
__device__ __forceinline__ void st4(T *p, const float (&v)[4]) {
    if constexpr (sizeof(T) == 2) {
        *reinterpret_cast<uint2 *>(p) = make_uint2(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]));
    } else {
        *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
    }
}

// The convolution for one (sequence, 4 channels): taps f(e, k) for channel c0+e.
template <typename T, int W, typename F>
__device__ __forceinline__ void decode_conv(const T *x_t, T *state, T *y_t, size_t b, int c0, int D, F f) {
    float x[4];
    ld4(x_t + b * D + c0, x);
    float win[W > 1 ? W - 1 : 1][4];     // win[i] = row i of the window (x_{t-(W-1)+i})
    T *st = state + b * (size_t)(W - 1) * D + c0;
#pragma unroll
    for (int i = 0; i < W - 1; ++i) ld4(st + (size_t)i * D, win[i]);
    float y[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        float acc = x[e];
        acc = fmaf(f(e, 0), x[e], acc);
#pragma unroll
        for (int k = 1; k < W; ++k) acc = fmaf(f(e, k), win[W - 1 - k][e], acc);
        y[e] = acc;
    }
    st4(y_t + b * D + c0, y);
#pragma unroll
    for (int i = 0; i + 1 < W - 1; ++i) st4(st + (size_t)i * D, win[i + 1]);
    if (W > 1) st4(st + (size_t)(W - 2) * D, x);
}

}  // namespace

// Low-rank decode: grid (D / 32, ceil(B / 32)).
template <typename T, int W>
__global__ void __launch_bounds__(kDcThreads)
k_decode_lowrank(const T *__restrict__ x_t, const T *__restrict__ z_t, const T *__restrict__ U,
                 T *__restrict__ state, T *__restrict__ y_t, int B, int D, int G, int R) {
    extern __shared__ float dsm[];
    const int N = (D / G) * W;
    const int cb = blockIdx.x * kDcCh;                 // first channel of the block
    const int ce = min(cb + kDcCh, D);
    const int b0 = blockIdx.y * kDcSeq;
    const int nb = min(kDcSeq, B - b0);
    const int g0 = cb / G, g1 = (ce - 1) / G;          // groups the block touches
    const int ncol = (g1 - g0 + 1) * W;                // their filter columns
    const int nq = (ncol + 3) / 4;                     // column quads
    float *zs = dsm;                                   // [R][32]  z^T of the block's sequences
    float *us = zs + R * kDcSeq;                       // [R][4*nq] U columns g0*W ..
    float *ws = us + R * 4 * nq;                       // [32][4*nq] w of the block
    const int tid = threadIdx.x;

    for (int e = tid; e < R * kDcSeq; e += kDcThreads) {
        const int r = e / kDcSeq, bl = e - r * kDcSeq;
        zs[e] = bl < nb ? to_f(z_t[(size_t)(b0 + bl) * R + r]) : 0.f;
    }
    if (sizeof(T) == 2 && ncol % 8 == 0 && (g0 * W) % 8 == 0 && N % 8 == 0) {
        // 8 columns per 16-byte load (the common case: the block's columns are aligned)
        const int n8 = ncol / 8;
        for (int e = tid; e < R * n8; e += kDcThreads) {
            const int r = e / n8, j8 = e - r * n8;
            const uint4 u = __ldg(reinterpret_cast<const uint4 *>(U + (size_t)r * N + g0 * W + 8 * j8));
            float *d = us + r * 4 * nq + 8 * j8;
            d[0] = bf16_lo(u.x); d[1] = bf16_hi(u.x); d[2] = bf16_lo(u.y); d[3] = bf16_hi(u.y);
            d[4] = bf16_lo(u.z); d[5] = bf16_hi(u.z); d[6] = bf16_lo(u.w); d[7] = bf16_hi(u.w);
        }
        for (int e = tid; e < R * (4 * nq - ncol); e += kDcThreads) {
            const int r = e / (4 * nq - ncol), j = ncol + e - r * (4 * nq - ncol);
            us[r * 4 * nq + j] = 0.f;
        }
    } else {
        for (int e = tid; e < R * 4 * nq; e += kDcThreads) {
            const int r = e / (4 * nq), j = e - r * 4 * nq;
            us[e] = j < ncol ? to_f(U[(size_t)r * N + g0 * W + j]) : 0.f;
        }
    }
    __syncthreads();
    // w[b, j] = sum_r z[b, r] U[r, j] in 4 (sequences) x 4 (columns) tiles
    for (int task = tid; task < (kDcSeq / 4) * nq; task += kDcThreads) {
        const int bq = task / nq, q = task - bq * nq;
        float acc[4][4] = {};
        for (int r = 0; r < R; ++r) {
            const float4 zv = *reinterpret_cast<const float4 *>(zs + r * kDcSeq + 4 * bq);
            const float4 uv = *reinterpret_cast<const float4 *>(us + r * 4 * nq + 4 * q);
            const float zz[4] = {zv.x, zv.y, zv.z, zv.w};
            const float uu[4] = {uv.x, uv.y, uv.z, uv.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) acc[i][jj] = fmaf(zz[i], uu[jj], acc[i][jj]);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
            *reinterpret_cast<float4 *>(ws + (4 * bq + i) * 4 * nq + 4 * q) =
                make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
    }
    __syncthreads();
    // convolution: thread = (sequence, 4 channels)
    const int nv = (ce - cb) / 4;
    for (int task = tid; task < nb * nv; task += kDcThreads) {
        const int bl = task / nv, v = task - bl * nv;
        const int c0 = cb + 4 * v;
        const float *wb = ws + bl * 4 * nq;
        decode_conv<T, W>(x_t, state, y_t, (size_t)(b0 + bl), c0, D,
                          [&](int e, int k) { return wb[((c0 + e) / G - g0) * W + k]; });
    }
}

// Low-rank decode for a few sequences (B <= kSmB): a block owns 64 channels; each thread
// forms 4 filter columns of them for every sequence straight from U in global memory
// (its R row loads are independent and issued together: one memory round trip, no U
// staging and no padded sequence rows), then the block applies the convolution, one
// thread per (sequence, 4 channels).  Needs the block's first column and N to be
// multiples of 4 (checked on the host).
constexpr int kSmCh = 64;          // channels per block
constexpr int kSmB = 4;            // largest batch
constexpr int kSmThreads = 128;

template <typename T, int W>
__global__ void __launch_bounds__(kSmThreads)
k_decode_lowrank_small(const T *__restrict__ x_t, const T *__restrict__ z_t, const T *__restrict__ U,
                       T *__restrict__ state, T *__restrict__ y_t, int B, int D, int G, int R) {
    extern __shared__ float dsm[];
    const int N = (D / G) * W;
    const int cb = blockIdx.x * kSmCh;
    const int ce = min(cb + kSmCh, D);
    const int g0 = cb / G, g1 = (ce - 1) / G;
    const int ncol = (g1 - g0 + 1) * W;                // this block's filter columns
    const int col0 = g0 * W;
    float *zs = dsm;                                   // [B][R]
    float *ws = zs + kSmB * R;                         // [B][ncol]
    const int tid = threadIdx.x;
    for (int e = tid; e < B * R; e += kSmThreads) zs[e] = to_f(z_t[e]);
    __syncthreads();
    for (int q = tid; 4 * q < ncol; q += kSmThreads) {
        float acc[kSmB][4] = {};
        const T *up = U + col0 + 4 * q;
#pragma unroll 16
        for (int r = 0; r < R; ++r) {
            float u[4];
            ld4(up + (size_t)r * N, u);
            float zb[kSmB];
#pragma unroll
            for (int b = 0; b < kSmB; ++b) zb[b] = b < B ? zs[b * R + r] : 0.f;
#pragma unroll
            for (int b = 0; b < kSmB; ++b)
#pragma unroll
                for (int i = 0; i < 4; ++i) acc[b][i] = fmaf(zb[b], u[i], acc[b][i]);
        }
#pragma unroll
        for (int b = 0; b < kSmB; ++b)
#pragma unroll
            for (int i = 0; i < 4; ++i)
                if (b < B && 4 * q + i < ncol) ws[b * ncol + 4 * q + i] = acc[b][i];
    }
    __syncthreads();
    const int nv = (ce - cb) / 4;
    for (int task = tid; task < B * nv; task += kSmThreads) {
        const int b = task / nv, v = task - b * nv;
        const int c0 = cb + 4 * v;
        const float *wb = ws + b * ncol;
        decode_conv<T, W>(x_t, state, y_t, (size_t)b, c0, D,
                          [&](int e, int k) { return wb[((c0 + e) / G - g0) * W + k]; });
    }
}

// Explicit-filter decode: w_t [B, D/G, W]; one thread per (sequence, 4 channels).
template <typename T, int W>
__global__ void __launch_bounds__(256)
k_decode(const T *__restrict__ x_t, const T *__restrict__ w_t, T *__restrict__ state, T *__restrict__ y_t, int B,
         int D, int G) {
    const int nv = D / 4;
    const size_t task = blockIdx.x * (size_t)blockDim.x + threadIdx.x;
    if (task >= (size_t)B * nv) return;
    const size_t b = task / nv;
    const int c0 = 4 * (int)(task - b * nv);
    const T *wb = w_t + b * (size_t)(D / G) * W;
    decode_conv<T, W>(x_t, state, y_t, b, c0, D, [&](int e, int k) { return to_f(wb[((c0 + e) / G) * W + k]); });
}

// ------------------------------------------------------------------ launchers
namespace {

size_t decode_smem(int D, int G, int W, int R) {
    // the widest block: 32 channels spanning (32 + G - 1) / G + 1 groups at most
    const int ng = std::min(D / G, (kDcCh + G - 1) / G + 1);
    const int nq = (ng * W + 3) / 4;
    return sizeof(float) * ((size_t)R * kDcSeq + (size_t)R * 4 * nq + (size_t)kDcSeq * 4 * nq);
}

// The small-batch kernel's conditions: at most kSmB sequences, a rank of at most 32 (a
// thread's R loads of U in flight at once; with R = 64 and 8 taps it measured slower,
// 5.49 -> 5.89 us at B = 1), whole 4-channel vectors per block, and filter columns that
// start every block (and every row of U) on a multiple of 4.  D=6144, R=32, W=4: B = 1
// 4.76 -> 3.79 us, B = 4 5.06 -> 3.83 us.
bool decode_small_ok(int B, int D, int G, int W, int R) {
    return B <= kSmB && R <= 32 && D % 4 == 0 && G <= kSmCh && kSmCh % G == 0 && ((kSmCh / G) * W) % 4 == 0 &&
           ((D / G) * W) % 4 == 0;
}
size_t decode_small_smem(int G, int W, int R) {
    return sizeof(float) * ((size_t)kSmB * R + (size_t)kSmB * (kSmCh / G + 1) * W);
}

template <typename T, int W>
cudaError_t launch_dl(const void *x, const void *z, const void *U, void *st, void *y, int B, int D, int G, int R,
                      cudaStream_t s) {
    if (decode_small_ok(B, D, G, W, R)) {
        const size_t smem = decode_small_smem(G, W, R);
        auto kern = k_decode_lowrank_small<T, W>;
        if (smem > 48 * 1024) {
            const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (e != cudaSuccess) return e;
        }
        kern<<<cdiv(D, kSmCh), kSmThreads, smem, s>>>((const T *)x, (const T *)z, (const T *)U, (T *)st, (T *)y,
                                                      B, D, G, R);
        return cudaGetLastError();
    }
    const size_t smem = decode_smem(D, G, W, R);
    auto kern = k_decode_lowrank<T, W>;
    if (smem > 48 * 1024) {
        const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    const dim3 grid(cdiv(D, kDcCh), cdiv(B, kDcSeq));
    kern<<<grid, kDcThreads, smem, s>>>((const T *)x, (const T *)z, (const T *)U, (T *)st, (T *)y, B, D, G, R);
    return cudaGetLastError();
}

template <typename T, int W>
cudaError_t launch_de(const void *x, const void *w, void *st, void *y, int B, int D, int G, cudaStream_t s) {
    const size_t n = (size_t)B * (D / 4);
    k_decode<T, W><<<(unsigned)((n + 255) / 256), 256, 0, s>>>((const T *)x, (const T *)w, (T *)st, (T *)y, B, D, G);
    return cudaGetLastError();
}

}  // namespace

bool decode_supported(int D, int G, int W, int R) { return decode_smem(D, G, W, R) <= 200 * 1024; }

cudaError_t launch_decode_lowrank(const void *x, const void *z, const void *U, void *st, void *y, int B, int D,
                                  int G, int W, int R, bool bf16_, cudaStream_t s) {
#define DSC_CASE(WW)                                                                                       \
    case WW:                                                                                               \
        return bf16_ ? launch_dl<bf16, WW>(x, z, U, st, y, B, D, G, R, s)                                  \
                     : launch_dl<float, WW>(x, z, U, st, y, B, D, G, R, s);
    switch (W) {
        DSC_CASE(1) DSC_CASE(2) DSC_CASE(3) DSC_CASE(4) DSC_CASE(5) DSC_CASE(6) DSC_CASE(7) DSC_CASE(8)
    }
#undef DSC_CASE
    return cudaErrorInvalidValue;
}

cudaError_t launch_decode(const void *x, const void *w, void *st, void *y, int B, int D, int G, int W, bool bf16_,
                          cudaStream_t s) {
#define DSC_CASE(WW)                                                                                       \
    case WW:                                                                                               \
        return bf16_ ? launch_de<bf16, WW>(x, w, st, y, B, D, G, s) : launch_de<float, WW>(x, w, st, y, B, D, G, s);
    switch (W) {
        DSC_CASE(1) DSC_CASE(2) DSC_CASE(3) DSC_CASE(4) DSC_CASE(5) DSC_CASE(6) DSC_CASE(7) DSC_CASE(8)
    }
#undef DSC_CASE
    return cudaErrorInvalidValue;
}

}  // namespace dsc
