// HBM-streaming CUDA-core kernels: the forward with static or explicit (head-wise tied)
// filters, and the static convolution's backward with dx and the filter gradient in
// one pass.
//
// "Convolucoes Curtas Dinamicas Melhoram Transformers": the static depthwise causal
// convolution is the primitive the method generalises (Declaracao do Problema), and
// Metodologia > Convolucoes Curtas Dinamicas defines the dynamic one,
//   y_t[c] = x_t[c] + sum_{k<W} f_t[c,k] x_{t-k}[c],   x_{t'} = 0 for t' < 0.
// These ops do 2-5 FLOP per byte; their bound is HBM bandwidth, and a kernel reaches it
// only with enough bytes in flight.  So a thread owns V channels (4 to 16 bytes of a
// token row) and walks a chunk of tokens of one sequence, keeping the W-1 rows it needs
// from earlier (or later) tokens in registers, and it loads the rows of U tokens at
// once before computing on them.  V shrinks as W grows, so that the filter taps and
// the row windows stay in registers with room for many resident warps.  A warp reads
// 32*V consecutive channels of a row, i.e. whole 128-byte lines.
#include "common.cuh"
#include "internal.h"

namespace dsc {

namespace {

template <int BYTES> struct RawOf;
template <> struct RawOf<4> { using type = uint32_t; };
template <> struct RawOf<8> { using type = uint2; };
template <> struct RawOf<16> { using type = uint4; };

// V elements of T held as raw 32-bit words (2 bf16 or 1 fp32 per word).
template <typename T, int V>
struct Pack {
    static constexpr int BYTES = V * (int)sizeof(T);
    static constexpr int WORDS = BYTES / 4;
    using raw_t = typename RawOf<BYTES>::type;

    __device__ __forceinline__ static raw_t load(const T *p) { return __ldg(reinterpret_cast<const raw_t *>(p)); }
    __device__ __forceinline__ static raw_t zero() {
        raw_t r;
        uint32_t *w = reinterpret_cast<uint32_t *>(&r);
#pragma unroll
        for (int i = 0; i < WORDS; ++i) w[i] = 0u;
        return r;
    }
    __device__ __forceinline__ static void unpack(const raw_t &r, float (&v)[V]) {
        const uint32_t *w = reinterpret_cast<const uint32_t *>(&r);
        if constexpr (sizeof(T) == 2) {
#pragma unroll
            for (int i = 0; i < WORDS; ++i) {
                v[2 * i] = bf16_lo(w[i]);
                v[2 * i + 1] = bf16_hi(w[i]);
            }
        } else {
#pragma unroll
            for (int i = 0; i < WORDS; ++i) v[i] = __uint_as_float(w[i]);
        }
    }
    __device__ __forceinline__ static void store(T *p, const float (&v)[V]) {
        raw_t r;
        uint32_t *w = reinterpret_cast<uint32_t *>(&r);
        if constexpr (sizeof(T) == 2) {
#pragma unroll
            for (int i = 0; i < WORDS; ++i) w[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
        } else {
#pragma unroll
            for (int i = 0; i < WORDS; ++i) w[i] = __float_as_uint(v[i]);
        }
        *reinterpret_cast<raw_t *>(p) = r;
    }
};

// Channels per thread: as many as keep the taps and row windows in registers.
template <typename T, int W>
struct Lanes {
    static constexpr int V = sizeof(T) == 2 ? (W <= 4 ? 4 : 2) : (W <= 4 ? 4 : 2);
};

constexpr int kU = 8;              // token rows loaded at once per thread
constexpr int kChunk = 128;        // tokens per thread (the W-1 row halo is re-read)
constexpr int kBX = 32;            // threads along channels (one warp)
constexpr int kBY = 8;             // chunks per block in the static backward

// Explicit per-token taps of V channels: w [B*T, D/G, W], element (bt, g, k).
template <typename T, int W, int V>
__device__ __forceinline__ void dyn_taps(const T *__restrict__ w, size_t bt, int c0, int D, int G,
                                         float (&f)[W][V]) {
    const int NG = D / G;
    if (G % V == 0) {
        const T *p = w + (bt * NG + c0 / G) * W;
        float t[W];
#pragma unroll
        for (int k = 0; k < W; ++k) t[k] = to_f(__ldg(p + k));
#pragma unroll
        for (int i = 0; i < V; ++i)
#pragma unroll
            for (int k = 0; k < W; ++k) f[k][i] = t[k];
    } else {
#pragma unroll
        for (int i = 0; i < V; ++i) {
            const T *p = w + (bt * NG + (c0 + i) / G) * W;
#pragma unroll
            for (int k = 0; k < W; ++k) f[k][i] = to_f(__ldg(p + k));
        }
    }
}

}  // namespace

// ------------------------------------------------------------------ forward
// y[t] = x[t] + sum_k f_t[k] x[t-k] for V channels over a chunk of tokens; f is the
// static w[c,k] (STATIC) or the explicit w[b,t,g(c),k].
template <typename T, int W, bool STATIC>
__global__ void __launch_bounds__(256)
k_stream_fwd(const T *__restrict__ x, const T *__restrict__ w, T *__restrict__ y, int B, int T_, int D,
             int G, int chunk) {
    constexpr int V = Lanes<T, W>::V;
    using P = Pack<T, V>;
    const int v = blockIdx.x * blockDim.x + threadIdx.x;
    if (v >= D / V) return;
    const int nch = cdiv(T_, chunk);
    const int b = blockIdx.y / nch;
    const int t0 = (blockIdx.y - b * nch) * chunk;
    const int t1 = min(t0 + chunk, T_);
    const int c0 = v * V;
    const T *xb = x + (size_t)b * T_ * D + c0;
    T *yb = y + (size_t)b * T_ * D + c0;

    float f[W][V];
    if (STATIC) {
#pragma unroll
        for (int i = 0; i < V; ++i)
#pragma unroll
            for (int k = 0; k < W; ++k) f[k][i] = to_f(__ldg(w + (size_t)(c0 + i) * W + k));
    }
    float win[W][V];   // win[k] = x[t-k]
#pragma unroll
    for (int k = 1; k < W; ++k) {
        if (t0 - k >= 0) P::unpack(P::load(xb + (size_t)(t0 - k) * D), win[k]);
        else
#pragma unroll
            for (int i = 0; i < V; ++i) win[k][i] = 0.f;
    }
    for (int tb = t0; tb < t1; tb += kU) {
        typename P::raw_t raw[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) raw[u] = (tb + u < t1) ? P::load(xb + (size_t)(tb + u) * D) : P::zero();
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const int t = tb + u;
            if (t >= t1) break;
            P::unpack(raw[u], win[0]);
            if (!STATIC) dyn_taps<T, W, V>(w, (size_t)b * T_ + t, c0, D, G, f);
            float out[V];
#pragma unroll
            for (int i = 0; i < V; ++i) {
                float acc = win[0][i];
#pragma unroll
                for (int k = 0; k < W; ++k) acc = fmaf(f[k][i], win[k][i], acc);
                out[i] = acc;
            }
            P::store(yb + (size_t)t * D, out);
#pragma unroll
            for (int k = W - 1; k >= 1; --k)
#pragma unroll
                for (int i = 0; i < V; ++i) win[k][i] = win[k - 1][i];
        }
    }
}

// ------------------------------------------------------------------ static backward
// One pass over x and dy per chunk of tokens:
//   dx[s]  = dy[s] + sum_k w[k] dy[s+k]             (dy rows t-k held in dyw[k])
//   dw[k] += dy[t] x[t-k]                            (x rows t-k held in xw[k])
// dx of row s = t-W+1 is complete at step t; W-1 extra steps past the chunk finish its
// last rows (reading the next chunk's first dy rows, or zeros past the sequence end).
// The block's kBY chunks sum their dw in shared memory in a fixed order and write one
// partial row part[p, c, k]; a second kernel adds the partials in order.
template <typename T, int W>
__global__ void __launch_bounds__(kBX * kBY)
k_static_bwd(const T *__restrict__ x, const T *__restrict__ ws, const T *__restrict__ dy, T *__restrict__ dx,
             float *__restrict__ part, int B, int T_, int D, int chunk) {
    constexpr int V = Lanes<T, W>::V;
    using P = Pack<T, V>;
    __shared__ float red[kBY][kBX][V];
    const int v = blockIdx.x * kBX + threadIdx.x;
    const bool active = v < D / V;
    const int nch = cdiv(T_, chunk);
    const int ngr = cdiv(nch, kBY);
    const int b = blockIdx.y / ngr;
    const int ci = (blockIdx.y - b * ngr) * kBY + threadIdx.y;
    const int t0 = ci * chunk;
    const int t1 = min(t0 + chunk, T_);
    const int c0 = v * V;
    const size_t off = (size_t)b * T_ * D + c0;

    float acc[W][V];
#pragma unroll
    for (int k = 0; k < W; ++k)
#pragma unroll
        for (int i = 0; i < V; ++i) acc[k][i] = 0.f;

    if (active && t0 < t1) {
        float f[W][V];
#pragma unroll
        for (int i = 0; i < V; ++i)
#pragma unroll
            for (int k = 0; k < W; ++k) f[k][i] = to_f(__ldg(ws + (size_t)(c0 + i) * W + k));
        float xw[W][V], dyw[W][V];
#pragma unroll
        for (int k = 1; k < W; ++k) {
#pragma unroll
            for (int i = 0; i < V; ++i) dyw[k][i] = 0.f;   // rows before t0 feed no dx row of this chunk
            if (t0 - k >= 0) P::unpack(P::load(x + off + (size_t)(t0 - k) * D), xw[k]);
            else
#pragma unroll
                for (int i = 0; i < V; ++i) xw[k][i] = 0.f;
        }
        auto step = [&](int t, bool in_chunk) {
            // dyw[0] and (in the chunk) xw[0] hold row t
            if (in_chunk) {
#pragma unroll
                for (int k = 0; k < W; ++k)
#pragma unroll
                    for (int i = 0; i < V; ++i) acc[k][i] = fmaf(dyw[0][i], xw[k][i], acc[k][i]);
            }
            const int s = t - (W - 1);
            if (s >= t0) {
                float o[V];
#pragma unroll
                for (int i = 0; i < V; ++i) {
                    float a = dyw[W - 1][i];
#pragma unroll
                    for (int k = 0; k < W; ++k) a = fmaf(f[k][i], dyw[W - 1 - k][i], a);
                    o[i] = a;
                }
                P::store(dx + off + (size_t)s * D, o);
            }
#pragma unroll
            for (int k = W - 1; k >= 1; --k)
#pragma unroll
                for (int i = 0; i < V; ++i) {
                    dyw[k][i] = dyw[k - 1][i];
                    xw[k][i] = xw[k - 1][i];
                }
        };
        for (int tb = t0; tb < t1; tb += kU) {
            typename P::raw_t rx[kU], rg[kU];
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const bool ok = tb + u < t1;
                rx[u] = ok ? P::load(x + off + (size_t)(tb + u) * D) : P::zero();
                rg[u] = ok ? P::load(dy + off + (size_t)(tb + u) * D) : P::zero();
            }
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                if (tb + u >= t1) break;
                P::unpack(rx[u], xw[0]);
                P::unpack(rg[u], dyw[0]);
                step(tb + u, true);
            }
        }
        // rows t1-W+1 .. t1-1 need dy rows t1 .. t1+W-2 (zero past the sequence end)
#pragma unroll
        for (int e = 0; e < W - 1; ++e) {
            const int t = t1 + e;
            if (t < T_) P::unpack(P::load(dy + off + (size_t)t * D), dyw[0]);
            else
#pragma unroll
                for (int i = 0; i < V; ++i) dyw[0][i] = 0.f;
            step(t, false);
        }
    }
#pragma unroll
    for (int k = 0; k < W; ++k) {
#pragma unroll
        for (int i = 0; i < V; ++i) red[threadIdx.y][threadIdx.x][i] = acc[k][i];
        __syncthreads();
        if (threadIdx.y == 0 && active) {
#pragma unroll
            for (int i = 0; i < V; ++i) {
                float s = 0.f;
#pragma unroll
                for (int yy = 0; yy < kBY; ++yy) s += red[yy][threadIdx.x][i];
                part[((size_t)blockIdx.y * D + c0 + i) * W + k] = s;
            }
        }
        __syncthreads();
    }
}

// out[e] = sum_{p < P} part[p * n + e], in order of p.
__global__ void k_sum_partials(const float *__restrict__ part, float *__restrict__ out, int P, size_t n) {
    for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < n; e += (size_t)gridDim.x * blockDim.x) {
        float s = 0.f;
        for (int p = 0; p < P; ++p) s += part[(size_t)p * n + e];
        out[e] = s;
    }
}

// ------------------------------------------------------------------ launchers
namespace {

int chunk_for(int T) { return T < kChunk ? T : kChunk; }

template <typename T, bool STATIC>
void launch_stream_fwd_T(const void *x, const void *w, void *y, int B, int T_, int D, int G, int W,
                         cudaStream_t s) {
    const int chunk = chunk_for(T_);
    const T *xp = (const T *)x;
    const T *wp = (const T *)w;
    T *yp = (T *)y;
    switch (W) {
#define DSC_CASE(WW)                                                                                  \
    case WW: {                                                                                        \
        constexpr int V = Lanes<T, WW>::V;                                                            \
        const dim3 grid(cdiv(D / V, 256), B * cdiv(T_, chunk));                                       \
        k_stream_fwd<T, WW, STATIC><<<grid, 256, 0, s>>>(xp, wp, yp, B, T_, D, G, chunk);             \
        break;                                                                                        \
    }
        DSC_CASE(1) DSC_CASE(2) DSC_CASE(3) DSC_CASE(4) DSC_CASE(5) DSC_CASE(6) DSC_CASE(7) DSC_CASE(8)
#undef DSC_CASE
    }
}

template <typename T>
void launch_static_bwd_T(const void *x, const void *w, const void *dy, void *dx, float *part, float *dw,
                         int B, int T_, int D, int W, cudaStream_t s) {
    const int chunk = chunk_for(T_);
    const int P = static_dw_partials(B, T_);
    const T *xp = (const T *)x;
    const T *wp = (const T *)w;
    const T *gp = (const T *)dy;
    T *op = (T *)dx;
    switch (W) {
#define DSC_CASE(WW)                                                                                  \
    case WW: {                                                                                        \
        constexpr int V = Lanes<T, WW>::V;                                                            \
        const dim3 grid(cdiv(D / V, kBX), P);                                                         \
        k_static_bwd<T, WW><<<grid, dim3(kBX, kBY), 0, s>>>(xp, wp, gp, op, part, B, T_, D, chunk);   \
        break;                                                                                        \
    }
        DSC_CASE(1) DSC_CASE(2) DSC_CASE(3) DSC_CASE(4) DSC_CASE(5) DSC_CASE(6) DSC_CASE(7) DSC_CASE(8)
#undef DSC_CASE
    }
    const size_t n = (size_t)D * W;
    const unsigned nb = (unsigned)std::min<size_t>((n + 255) / 256, 4096);
    k_sum_partials<<<nb, 256, 0, s>>>(part, dw, P, n);
}

}  // namespace

int static_dw_partials(int B, int T) { return B * cdiv(cdiv(T, chunk_for(T)), kBY); }

void launch_conv_fwd(const void *x, const void *w, void *y, int B, int T, int D, int G, int W, bool bf16_,
                     bool is_static, cudaStream_t s) {
    if (bf16_) {
        if (is_static) launch_stream_fwd_T<bf16, true>(x, w, y, B, T, D, 1, W, s);
        else launch_stream_fwd_T<bf16, false>(x, w, y, B, T, D, G, W, s);
    } else {
        if (is_static) launch_stream_fwd_T<float, true>(x, w, y, B, T, D, 1, W, s);
        else launch_stream_fwd_T<float, false>(x, w, y, B, T, D, G, W, s);
    }
}

void launch_static_bwd(const void *x, const void *w, const void *dy, void *dx, float *part, float *dw, int B,
                       int T, int D, int W, bool bf16_, cudaStream_t s) {
    if (bf16_) launch_static_bwd_T<bf16>(x, w, dy, dx, part, dw, B, T, D, W, s);
    else launch_static_bwd_T<float>(x, w, dy, dx, part, dw, B, T, D, W, s);
}

}  // namespace dsc
