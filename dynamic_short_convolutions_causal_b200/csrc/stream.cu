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
// from earlier (or later) tokens in registers.  Its rows arrive a batch of 8 or 16
// tokens at a time through shared memory with cp.async, double-buffered: the next batch is in
// flight while the current one is used, and the bytes in flight cost no registers.  A
// warp reads 32*V consecutive channels of a row (whole 128-byte lines), and the
// staging layout interleaves the threads so that their shared-memory reads do not
// conflict.  V shrinks as W grows, so that the taps and row windows stay in registers.
// Two things keep the instruction count and the registers down (measured on B200):
//   - bf16 rows and taps stay packed, two channels a word, and every product is a
//     mixed fma.rn.f32.bf16 (exact product, one rounding: the results of widening
//     first): 8-tap static forward of the MLP-width shape 0.133 -> 0.111 ms, its
//     backward 0.272 -> 0.222 ms, tied-filter forward / backward of the stacked-QKV
//     shape 0.083 -> 0.074 / 0.162 -> 0.143 ms;
//   - the row window is a ring when a batch is a whole number of windows: row t sits
//     in slot (t - t0) % W, a constant in each unrolled step, so no row is copied
//     (0.141 -> 0.134 ms and 0.283 -> 0.272 ms on the static forward / backward).
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

// Channels per thread: 16 bytes of a bf16 row for up to 4 taps, 8 bytes for more, as many
// as keep the taps and row windows in registers (measured on B200: the tied-filter
// forward of the stacked-QKV shape 0.140 -> 0.085 ms going from 8 to 16 bytes, the
// 8-tap static forward of the MLP-width shape 0.163 -> 0.142 ms from 4 to 8 bytes).
template <typename T, int W>
struct Lanes {
    static constexpr int V = sizeof(T) == 2 ? (W <= 4 ? 8 : 4) : (W <= 4 ? 4 : 2);
};

constexpr int kChunk = 128;        // tokens per thread in the backward (the W-1 row halos are re-read)
constexpr int kChunkFwd = 32;      // in the forward: more, shorter token walks in parallel
constexpr int kBX = 32;            // threads along channels (one warp)
constexpr int kBY = 4;             // chunks per block in the static backward (128-thread blocks:
                                   // three fit an SM at its 160 registers a thread; 8 chunks,
                                   // one block an SM: 0.222 -> 0.200 ms on the MLP-width shape)

__host__ __device__ inline int chunk_for(int T) { return T < kChunk ? T : kChunk; }
// tokens per thread in the forward: short walks for few taps (more walks in parallel),
// long ones for many taps (the W-1 halo rows each walk re-reads)
inline int chunk_fwd(int T, int W) {
    const int c = W <= 4 ? kChunkFwd : kChunk;
    return T < c ? T : c;
}
__host__ __device__ inline int dw_partials(int B, int T) { return B * cdiv(cdiv(T, chunk_for(T)), kBY); }

// cp.async of BYTES (4, 8 or 16) from global to shared memory; when `valid` is false the
// destination is zero-filled and nothing is read.
template <int BYTES>
__device__ __forceinline__ void cp_async(uint32_t dst, const void *src, bool valid) {
    const int n = valid ? BYTES : 0;
    if constexpr (BYTES == 16)
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
    else
        asm volatile("cp.async.ca.shared.global [%0], [%1], %2, %3;" ::"r"(dst), "l"(src), "n"(BYTES), "r"(n)
                     : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

template <typename R>
__device__ __forceinline__ R lds_raw(uint32_t addr) {
    R r;
    if constexpr (sizeof(R) == 4) {
        asm volatile("ld.shared.u32 %0, [%1];" : "=r"(r) : "r"(addr));
    } else if constexpr (sizeof(R) == 8) {
        asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(r.x), "=r"(r.y) : "r"(addr));
    } else {
        asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "r"(addr));
    }
    return r;
}

// Shared-memory staging of a thread's row batches: slot (stage, tensor, row u) of thread
// `tid` is at ((stage * NT + tensor) * KU + u) * NTHREADS * BYTES + tid * BYTES.
template <int BYTES, int NT, int KU, int NTHREADS = 256>
struct Staging {
    uint32_t base;            // this thread's slot 0: block base + tid * BYTES
    __device__ Staging(uint32_t block_base, int tid) : base(block_base + (uint32_t)(tid * BYTES)) {}
    __device__ uint32_t at(int stage, int tensor, int u) const {
        return base + (uint32_t)(((stage * NT + tensor) * KU + u) * NTHREADS * BYTES);
    }
    static constexpr int bytes_per_thread() { return 2 * NT * KU * BYTES; }
};

// Rows per batch: 64 bytes of each staged tensor per thread and batch (16 rows of 4
// bytes, 8 of 8, 4 of 16), which keeps a block's staging at or below 64 KB so that
// several blocks share an SM.
template <int SLOT> struct Batch { static constexpr int KU = 64 / SLOT; };

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
// static w[c,k] (STATIC) or the explicit w[b,t,g(c),k].  With explicit filters whose
// group covers the thread's V channels (G % V == 0) and whose W taps make a 4-, 8- or
// 16-byte aligned vector, the taps are staged with the rows; otherwise they are read
// per token.
template <typename T, int W, bool STATIC>
__device__ __forceinline__ void stream_fwd_item(const T *__restrict__ x, const T *__restrict__ w, T *__restrict__ y,
                                                int B, int T_, int D, int G, int chunk, int bx, int by) {
    constexpr int V = Lanes<T, W>::V;
    using P = Pack<T, V>;
    constexpr int TB = W * (int)sizeof(T);                         // bytes of one token's taps
    constexpr bool kTapVec = !STATIC && (TB == 4 || TB == 8 || TB == 16);
    constexpr int NT = kTapVec ? 2 : 1;
    constexpr int SB = P::BYTES > TB || !kTapVec ? P::BYTES : TB;  // slot size
    constexpr int KU = Batch<SB>::KU;
    extern __shared__ __align__(16) uint8_t stg_raw[];
    const Staging<SB, NT, KU> stg((uint32_t)__cvta_generic_to_shared(stg_raw), (int)threadIdx.x);
    const int v = bx * 256 + threadIdx.x;
    const bool active = v < D / V;
    const int nch = cdiv(T_, chunk);
    const int b = by / nch;
    const int t0 = (by - b * nch) * chunk;
    const int t1 = min(t0 + chunk, T_);
    const int c0 = active ? v * V : 0;
    const T *xb = x + (size_t)b * T_ * D + c0;
    T *yb = y + (size_t)b * T_ * D + c0;
    const bool tap_stage = kTapVec && (G % V == 0);
    const T *wb = STATIC ? w : w + ((size_t)b * T_ * (D / G) + c0 / G) * W;   // taps of token 0
    auto issue = [&](int tb, int stage) {
#pragma unroll
        for (int u = 0; u < KU; ++u) {
            const bool ok = active && tb + u < t1;
            const int t = ok ? tb + u : t0;
            cp_async<P::BYTES>(stg.at(stage, 0, u), xb + (size_t)t * D, ok);
            if constexpr (kTapVec)
                if (tap_stage) cp_async<TB>(stg.at(stage, 1, u), wb + (size_t)t * (D / G) * W, ok);
        }
        cp_commit();
    };
    // The W-row window.  When a batch is a whole number of windows (KU % W == 0) and the
    // chunk starts at a multiple of W, row t sits in slot t % W, a constant in every
    // unrolled step, so no row is copied (ring); otherwise win[k] = x[t-k] and the rows
    // move down one slot per token (shift).
    constexpr bool kRing = KU % W == 0;
    const bool ring = kRing && t0 % W == 0;
    const int nb = cdiv(t1 - t0, KU);

    if constexpr (sizeof(T) == 2) {
        if (STATIC || tap_stage) {
            // bf16 with static or staged taps: rows and taps stay packed (two channels a
            // word) and every product is a mixed fma.rn.f32.bf16 (exact product, one
            // rounding: the results of widening first), fewer registers and no unpacking
            constexpr int NW = V / 2;
            using RT = typename P::raw_t;
            auto words = [](const RT &r, uint32_t (&o)[NW]) {
                const uint32_t *q = reinterpret_cast<const uint32_t *>(&r);
#pragma unroll
                for (int j = 0; j < NW; ++j) o[j] = q[j];
            };
            uint32_t fw[W][NW];      // static taps of channel pairs (w[c0+2j, k], w[c0+2j+1, k])
            if (STATIC && active) {
                const uint16_t *wr = reinterpret_cast<const uint16_t *>(w);
#pragma unroll
                for (int j = 0; j < NW; ++j)
#pragma unroll
                    for (int k = 0; k < W; ++k)
                        fw[k][j] = (uint32_t)__ldg(wr + (size_t)(c0 + 2 * j) * W + k) |
                                   ((uint32_t)__ldg(wr + (size_t)(c0 + 2 * j + 1) * W + k) << 16);
            }
            uint32_t win[W][NW];
#pragma unroll
            for (int k = 1; k < W; ++k) {
                uint32_t r[NW];
                if (active && t0 - k >= 0) words(P::load(xb + (size_t)(t0 - k) * D), r);
                else
#pragma unroll
                    for (int j = 0; j < NW; ++j) r[j] = 0u;
                const int sk = (kRing && ring) ? W - k : k;
#pragma unroll
                for (int j = 0; j < NW; ++j) win[sk][j] = r[j];
            }
            issue(t0, 0);
            for (int bi = 0; bi < nb; ++bi) {
                const int tb = t0 + bi * KU, stage = bi & 1;
                if (bi + 1 < nb) issue(tb + KU, stage ^ 1);
                else cp_commit();
                cp_wait<1>();
                if (!active) continue;
                auto token = [&](int t, int u, auto sl) {
                    words(lds_raw<RT>(stg.at(stage, 0, u)), win[sl(0)]);
                    uint32_t tw[TB / 4 > 0 ? TB / 4 : 1];          // the token's taps, two a word
                    (void)tw;
                    if constexpr (kTapVec) {
                        if (!STATIC) {
                            using TR = typename RawOf<TB>::type;
                            const TR tr = lds_raw<TR>(stg.at(stage, 1, u));
                            const uint32_t *q = reinterpret_cast<const uint32_t *>(&tr);
#pragma unroll
                            for (int m = 0; m < TB / 4; ++m) tw[m] = q[m];
                        }
                    }
                    float out[V];
#pragma unroll
                    for (int j = 0; j < NW; ++j) {
                        const uint32_t xt = win[sl(0)][j];
                        float a0 = bf16_lo(xt), a1 = bf16_hi(xt);
#pragma unroll
                        for (int k = 0; k < W; ++k) {
                            const uint32_t xk = win[sl(k)][j];
                            if constexpr (STATIC) {
                                a0 = fma_bf16_sel<0, 0>(fw[k][j], xk, a0);
                                a1 = fma_bf16_sel<1, 1>(fw[k][j], xk, a1);
                            } else if ((k & 1) == 0) {
                                a0 = fma_bf16_sel<0, 0>(tw[k / 2], xk, a0);
                                a1 = fma_bf16_sel<0, 1>(tw[k / 2], xk, a1);
                            } else {
                                a0 = fma_bf16_sel<1, 0>(tw[k / 2], xk, a0);
                                a1 = fma_bf16_sel<1, 1>(tw[k / 2], xk, a1);
                            }
                        }
                        out[2 * j] = a0;
                        out[2 * j + 1] = a1;
                    }
                    P::store(yb + (size_t)t * D, out);
                };
                if (kRing && ring) {
#pragma unroll
                    for (int u = 0; u < KU; ++u) {
                        const int t = tb + u;
                        if (t >= t1) break;
                        token(t, u, [&](int k) { return (u - k + W) % W; });
                    }
                } else {
#pragma unroll
                    for (int u = 0; u < KU; ++u) {
                        const int t = tb + u;
                        if (t >= t1) break;
                        token(t, u, [](int k) { return k; });
#pragma unroll
                        for (int k = W - 1; k >= 1; --k)
#pragma unroll
                            for (int j = 0; j < NW; ++j) win[k][j] = win[k - 1][j];
                    }
                }
            }
            cp_wait<0>();
            return;
        }
    }

    float f[W][V];
    if (STATIC && active) {
#pragma unroll
        for (int i = 0; i < V; ++i)
#pragma unroll
            for (int k = 0; k < W; ++k) f[k][i] = to_f(__ldg(w + (size_t)(c0 + i) * W + k));
    }
    float win[W][V];
#pragma unroll
    for (int k = 1; k < W; ++k) {
        float r[V];
        if (active && t0 - k >= 0) P::unpack(P::load(xb + (size_t)(t0 - k) * D), r);
        else
#pragma unroll
            for (int i = 0; i < V; ++i) r[i] = 0.f;
        // row t0-k: slot (t0-k) % W = W-k in the ring, k in the shift
        if (kRing && ring) {
#pragma unroll
            for (int i = 0; i < V; ++i) win[W - k][i] = r[i];
        } else {
#pragma unroll
            for (int i = 0; i < V; ++i) win[k][i] = r[i];
        }
    }
    issue(t0, 0);
    for (int bi = 0; bi < nb; ++bi) {
        const int tb = t0 + bi * KU, stage = bi & 1;
        if (bi + 1 < nb) issue(tb + KU, stage ^ 1);
        else cp_commit();
        cp_wait<1>();
        if (!active) continue;
        // y[t] from the window (slot of row t-k: sl(k)) and the token's taps
        auto token = [&](int t, int u, auto sl) {
            P::unpack(lds_raw<typename P::raw_t>(stg.at(stage, 0, u)), win[sl(0)]);
            if constexpr (!STATIC) {
                bool staged = false;
                if constexpr (kTapVec) {
                    if (tap_stage) {
                        staged = true;
                        using TR = typename RawOf<TB>::type;
                        const TR tr = lds_raw<TR>(stg.at(stage, 1, u));
                        uint32_t tw[TB / 4];
                        if constexpr (TB == 4) {
                            tw[0] = tr;
                        } else if constexpr (TB == 8) {
                            tw[0] = tr.x; tw[1] = tr.y;
                        } else {
                            tw[0] = tr.x; tw[1] = tr.y; tw[2] = tr.z; tw[3] = tr.w;
                        }
#pragma unroll
                        for (int k = 0; k < W; ++k) {
                            float fk;
                            if constexpr (sizeof(T) == 2) fk = (k & 1) ? bf16_hi(tw[k / 2]) : bf16_lo(tw[k / 2]);
                            else fk = __uint_as_float(tw[k]);
#pragma unroll
                            for (int i = 0; i < V; ++i) f[k][i] = fk;
                        }
                    }
                }
                if (!staged) dyn_taps<T, W, V>(w, (size_t)b * T_ + t, c0, D, G, f);
            }
            float out[V];
#pragma unroll
            for (int i = 0; i < V; ++i) {
                float acc = win[sl(0)][i];
#pragma unroll
                for (int k = 0; k < W; ++k) acc = fmaf(f[k][i], win[sl(k)][i], acc);
                out[i] = acc;
            }
            P::store(yb + (size_t)t * D, out);
        };
        if (kRing && ring) {
#pragma unroll
            for (int u = 0; u < KU; ++u) {
                const int t = tb + u;
                if (t >= t1) break;
                token(t, u, [&](int k) { return (u - k + W) % W; });
            }
        } else {
#pragma unroll
            for (int u = 0; u < KU; ++u) {
                const int t = tb + u;
                if (t >= t1) break;
                token(t, u, [](int k) { return k; });
#pragma unroll
                for (int k = W - 1; k >= 1; --k)
#pragma unroll
                    for (int i = 0; i < V; ++i) win[k][i] = win[k - 1][i];
            }
        }
    }
    cp_wait<0>();
}

template <typename T, int W, bool STATIC>
__global__ void __launch_bounds__(256)
k_stream_fwd(const T *__restrict__ x, const T *__restrict__ w, T *__restrict__ y, int B, int T_, int D,
             int G, int chunk) {
    // work item = 256 thread-vectors of channels x one chunk of one sequence; the grid
    // has one block per item (the loop also serves smaller grids)
    constexpr int V0 = Lanes<T, W>::V;
    const int nbx = cdiv(D / V0, 256);
    const int nitems = nbx * B * cdiv(T_, chunk);
    for (int item = blockIdx.x; item < nitems; item += gridDim.x)
        stream_fwd_item<T, W, STATIC>(x, w, y, B, T_, D, G, chunk, item % nbx, item / nbx);
}


// ------------------------------------------------------------------ explicit backward
// One pass over x, dy and the per-token taps of a chunk of tokens (dx in scatter form):
//   token t adds dy[t] (the residual) and w[t,g,k] dy[t] into the open dx row t-k; row
//   t-W+1 is then complete; W-1 tokens past the chunk finish its last rows;
//   dw[t,g,k] = sum_{c in g} dy[t,c] x[t-k,c]: the thread's V channels are summed in the
//   thread and across the G/V threads of a group by a fixed xor-shuffle tree.
// Taken when the taps are staged with the rows (W * sizeof(T) of 4, 8 or 16 bytes) and
// the groups tile the threads' channel vectors (G % V == 0, G/V a power of two <= 32).
template <typename T, int W>
__global__ void __launch_bounds__(256)
k_dyn_bwd(const T *__restrict__ x, const T *__restrict__ w, const T *__restrict__ dy, T *__restrict__ dx,
          float *__restrict__ dw, int B, int T_, int D, int G, int chunk) {
    constexpr int V = Lanes<T, W>::V;
    using P = Pack<T, V>;
    constexpr int TB = W * (int)sizeof(T);                         // bytes of one token's taps
    constexpr int SB = P::BYTES > TB ? P::BYTES : TB;              // slot size
    constexpr int KU = Batch<SB>::KU;
    using TR = typename RawOf<TB>::type;
    extern __shared__ __align__(16) uint8_t stg_raw[];
    const Staging<SB, 3, KU> stg((uint32_t)__cvta_generic_to_shared(stg_raw), (int)threadIdx.x);
    const int nbx = cdiv(D / V, 256);
    const int nch = cdiv(T_, chunk);
    const int nitems = nbx * B * nch;
    const int NG = D / G;
    const int lanes = G / V;
    for (int item = blockIdx.x; item < nitems; item += gridDim.x) {
        const int bx = item % nbx, by = item / nbx;
        const int v = bx * 256 + threadIdx.x;
        const bool active = v < D / V;
        const int b = by / nch;
        const int t0 = (by - b * nch) * chunk;
        const int t1 = min(t0 + chunk, T_);
        const int t1e = min(t1 + W - 1, T_);         // dy and taps needed up to here
        const int c0 = active ? v * V : 0;
        const size_t row0 = (size_t)b * T_;
        const T *xb = x + row0 * D + c0;
        const T *gb = dy + row0 * D + c0;
        T *ob = dx + row0 * D + c0;
        const T *wb = w + (row0 * NG + c0 / G) * W;
        if constexpr (sizeof(T) == 2) {
            // bf16: rows and taps stay packed (two channels a word), every product is a
            // mixed fma.rn.f32.bf16 (the results of widening first).  Windows: a ring
            // (row r in slot (r - t0) % W, constant in every unrolled step) when a batch is
            // a whole number of windows, else shifted one slot per token.
            constexpr int NW = V / 2;
            using RT = typename P::raw_t;
            auto words = [](const RT &r, uint32_t (&o)[NW]) {
                const uint32_t *q = reinterpret_cast<const uint32_t *>(&r);
#pragma unroll
                for (int j = 0; j < NW; ++j) o[j] = q[j];
            };
            constexpr bool kRing = KU % W == 0;
            const bool ring = kRing && t0 % W == 0;
            float acc[W][V];                         // open dx rows (slot of row t-k: sl(k))
            uint32_t xw[W][NW];                      // x rows, packed
#pragma unroll
            for (int k = 0; k < W; ++k)
#pragma unroll
                for (int i = 0; i < V; ++i) acc[k][i] = 0.f;
#pragma unroll
            for (int k = 1; k < W; ++k) {
                uint32_t r[NW];
                if (active && t0 - k >= 0) words(P::load(xb + (size_t)(t0 - k) * D), r);
                else
#pragma unroll
                    for (int j = 0; j < NW; ++j) r[j] = 0u;
                const int sk = (kRing && ring) ? W - k : k;
#pragma unroll
                for (int j = 0; j < NW; ++j) xw[sk][j] = r[j];
            }
            auto issue = [&](int tb, int stage) {
#pragma unroll
                for (int u = 0; u < KU; ++u) {
                    const bool ok = active && tb + u < t1e;
                    const int t = ok ? tb + u : t0;
                    cp_async<P::BYTES>(stg.at(stage, 0, u), xb + (size_t)t * D, ok && tb + u < t1);
                    cp_async<P::BYTES>(stg.at(stage, 1, u), gb + (size_t)t * D, ok);
                    cp_async<TB>(stg.at(stage, 2, u), wb + (size_t)t * NG * W, ok);
                }
                cp_commit();
            };
            // token t: its rows and taps from the stage; sl(k) is the slot of row t-k
            auto token = [&](int t, int stage, int u, auto sl) {
                uint32_t gw[NW], tw[TB / 4];
                words(lds_raw<RT>(stg.at(stage, 1, u)), gw);
                words(lds_raw<RT>(stg.at(stage, 0, u)), xw[sl(0)]);
                {
                    const TR tr = lds_raw<TR>(stg.at(stage, 2, u));
                    const uint32_t *q = reinterpret_cast<const uint32_t *>(&tr);
#pragma unroll
                    for (int m = 0; m < TB / 4; ++m) tw[m] = q[m];
                }
                // dx: row t opens with dy[t] (its slot held row t-W, stored a step ago),
                // every open row t-k gets w[t,k] dy[t]; row t-W+1 is then complete
#pragma unroll
                for (int j = 0; j < NW; ++j) {
                    acc[sl(0)][2 * j] = bf16_lo(gw[j]);
                    acc[sl(0)][2 * j + 1] = bf16_hi(gw[j]);
                }
#pragma unroll
                for (int k = 0; k < W; ++k)
#pragma unroll
                    for (int j = 0; j < NW; ++j) {
                        float &a0 = acc[sl(k)][2 * j], &a1 = acc[sl(k)][2 * j + 1];
                        if ((k & 1) == 0) {
                            a0 = fma_bf16_sel<0, 0>(tw[k / 2], gw[j], a0);
                            a1 = fma_bf16_sel<0, 1>(tw[k / 2], gw[j], a1);
                        } else {
                            a0 = fma_bf16_sel<1, 0>(tw[k / 2], gw[j], a0);
                            a1 = fma_bf16_sel<1, 1>(tw[k / 2], gw[j], a1);
                        }
                    }
                const int s = t - (W - 1);
                if (active && s >= t0 && s < t1) P::store(ob + (size_t)s * D, acc[sl(W - 1)]);
                // dw of token t (tokens of the chunk only)
                if (t < t1) {
                    float sw[W];
#pragma unroll
                    for (int k = 0; k < W; ++k) {
                        float a = 0.f;
#pragma unroll
                        for (int j = 0; j < NW; ++j) {
                            a = fma_bf16_sel<0, 0>(gw[j], xw[sl(k)][j], a);
                            a = fma_bf16_sel<1, 1>(gw[j], xw[sl(k)][j], a);
                        }
                        sw[k] = a;
                    }
                    for (int o = 1; o < lanes; o <<= 1)
#pragma unroll
                        for (int k = 0; k < W; ++k) sw[k] += __shfl_xor_sync(0xffffffffu, sw[k], o);
                    if (active && (v % lanes) == 0) {
                        float *q = dw + ((row0 + t) * NG + c0 / G) * W;
#pragma unroll
                        for (int k = 0; k < W; ++k) q[k] = sw[k];
                    }
                }
            };
            const int nb = cdiv(t1e - t0, KU);
            issue(t0, 0);
            for (int bi = 0; bi < nb; ++bi) {
                const int tb = t0 + bi * KU, stage = bi & 1;
                if (bi + 1 < nb) issue(tb + KU, stage ^ 1);
                else cp_commit();
                cp_wait<1>();
                if (kRing && ring) {
#pragma unroll
                    for (int u = 0; u < KU; ++u) {
                        if (tb + u >= t1e) break;
                        token(tb + u, stage, u, [&](int k) { return (u - k + W) % W; });
                    }
                } else {
#pragma unroll
                    for (int u = 0; u < KU; ++u) {
                        if (tb + u >= t1e) break;
                        // open rows move down before the token (slot 0 is row t), x rows
                        // after it (xw[k] = x[t-k] while the token runs)
#pragma unroll
                        for (int k = W - 1; k >= 1; --k)
#pragma unroll
                            for (int i = 0; i < V; ++i) acc[k][i] = acc[k - 1][i];
                        token(tb + u, stage, u, [](int k) { return k; });
#pragma unroll
                        for (int k = W - 1; k >= 1; --k)
#pragma unroll
                            for (int j = 0; j < NW; ++j) xw[k][j] = xw[k - 1][j];
                    }
                }
            }
            cp_wait<0>();
            // at the sequence end the rows still open have all their contributions: rows
            // T-W+1 .. T-1, in slots (row - t0) % W (ring) or T-1-row (shift)
            if (t1e == T_) {
                auto store_open = [&](auto sl_of_row) {
#pragma unroll
                    for (int k = 1; k < W; ++k) {
                        const int s = T_ - W + k;
                        if (active && s >= t0 && s < t1) P::store(ob + (size_t)s * D, acc[sl_of_row(k)]);
                    }
                };
                if (kRing && ring) {
                    // slot of row T-W+k is (T - t0 - W + k) % W = (p + k) % W, p = (T - t0) % W
                    const int p = (T_ - t0) % W;
#pragma unroll
                    for (int pp = 0; pp < W; ++pp)
                        if (pp == p) store_open([&](int k) { return (pp + k) % W; });
                } else {
                    store_open([](int k) { return W - 1 - k; });   // row T-W+k = (T-1) - (W-1-k)
                }
            }
        } else {
        float acc[W][V];                             // acc[k] = open dx row t-k
        float xw[W][V];                              // xw[k] = x[t-k]
#pragma unroll
        for (int k = 0; k < W; ++k)
#pragma unroll
            for (int i = 0; i < V; ++i) acc[k][i] = 0.f;
#pragma unroll
        for (int k = 1; k < W; ++k) {
            if (active && t0 - k >= 0) P::unpack(P::load(xb + (size_t)(t0 - k) * D), xw[k]);
            else
#pragma unroll
                for (int i = 0; i < V; ++i) xw[k][i] = 0.f;
        }
        auto issue = [&](int tb, int stage) {
#pragma unroll
            for (int u = 0; u < KU; ++u) {
                const bool ok = active && tb + u < t1e;
                const int t = ok ? tb + u : t0;
                cp_async<P::BYTES>(stg.at(stage, 0, u), xb + (size_t)t * D, ok && tb + u < t1);
                cp_async<P::BYTES>(stg.at(stage, 1, u), gb + (size_t)t * D, ok);
                cp_async<TB>(stg.at(stage, 2, u), wb + (size_t)t * NG * W, ok);
            }
            cp_commit();
        };
        const int nb = cdiv(t1e - t0, KU);
        issue(t0, 0);
        for (int bi = 0; bi < nb; ++bi) {
            const int tb = t0 + bi * KU, stage = bi & 1;
            if (bi + 1 < nb) issue(tb + KU, stage ^ 1);
            else cp_commit();
            cp_wait<1>();
#pragma unroll
            for (int u = 0; u < KU; ++u) {
                const int t = tb + u;
                if (t >= t1e) break;
                float g[V];
                P::unpack(lds_raw<typename P::raw_t>(stg.at(stage, 1, u)), g);
                P::unpack(lds_raw<typename P::raw_t>(stg.at(stage, 0, u)), xw[0]);
                const TR tr = lds_raw<TR>(stg.at(stage, 2, u));
                uint32_t tw[TB / 4];
                if constexpr (TB == 4) {
                    tw[0] = tr;
                } else if constexpr (TB == 8) {
                    tw[0] = tr.x; tw[1] = tr.y;
                } else {
                    tw[0] = tr.x; tw[1] = tr.y; tw[2] = tr.z; tw[3] = tr.w;
                }
                float f[W];
#pragma unroll
                for (int k = 0; k < W; ++k) {
                    if constexpr (sizeof(T) == 2) f[k] = (k & 1) ? bf16_hi(tw[k / 2]) : bf16_lo(tw[k / 2]);
                    else f[k] = __uint_as_float(tw[k]);
                }
                // dx: open row t; add token t's contributions; row t-W+1 is complete
#pragma unroll
                for (int k = W - 1; k >= 1; --k)
#pragma unroll
                    for (int i = 0; i < V; ++i) acc[k][i] = acc[k - 1][i];
#pragma unroll
                for (int i = 0; i < V; ++i) acc[0][i] = g[i];
#pragma unroll
                for (int k = 0; k < W; ++k)
#pragma unroll
                    for (int i = 0; i < V; ++i) acc[k][i] = fmaf(f[k], g[i], acc[k][i]);
                const int s = t - (W - 1);
                if (active && s >= t0 && s < t1) P::store(ob + (size_t)s * D, acc[W - 1]);
                // dw of token t (tokens of the chunk only)
                if (t < t1) {
                    float sw[W];
#pragma unroll
                    for (int k = 0; k < W; ++k) {
                        float a = 0.f;
#pragma unroll
                        for (int i = 0; i < V; ++i) a = fmaf(g[i], xw[k][i], a);
                        sw[k] = a;
                    }
                    for (int o = 1; o < lanes; o <<= 1)
#pragma unroll
                        for (int k = 0; k < W; ++k) sw[k] += __shfl_xor_sync(0xffffffffu, sw[k], o);
                    if (active && (v % lanes) == 0) {
                        float *q = dw + ((row0 + t) * NG + c0 / G) * W;
#pragma unroll
                        for (int k = 0; k < W; ++k) q[k] = sw[k];
                    }
                }
#pragma unroll
                for (int k = W - 1; k >= 1; --k)
#pragma unroll
                    for (int i = 0; i < V; ++i) xw[k][i] = xw[k - 1][i];
            }
        }
        cp_wait<0>();
        // at the sequence end the rows still open have all their contributions
        if (t1e == T_) {
#pragma unroll
            for (int k = 1; k < W; ++k) {
#pragma unroll
                for (int kk = W - 1; kk >= 1; --kk)
#pragma unroll
                    for (int i = 0; i < V; ++i) acc[kk][i] = acc[kk - 1][i];
#pragma unroll
                for (int i = 0; i < V; ++i) acc[0][i] = 0.f;
                const int s = T_ - 1 - (W - 1) + k;      // row completed by this virtual step
                if (active && s >= t0 && s < t1) P::store(ob + (size_t)s * D, acc[W - 1]);
            }
        }
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
__device__ __forceinline__ void static_bwd_item(const T *__restrict__ x, const T *__restrict__ ws,
                                                const T *__restrict__ dy, T *__restrict__ dx,
                                                float *__restrict__ part, int B, int T_, int D, int chunk,
                                                int bx, int by) {
    constexpr int V = Lanes<T, W>::V;
    using P = Pack<T, V>;
    constexpr int kU = Batch<P::BYTES>::KU;
    __shared__ float red[kBY][kBX][V];
    extern __shared__ __align__(16) uint8_t stg_raw[];
    const int v = bx * kBX + threadIdx.x;
    const bool active = v < D / V;
    const int nch = cdiv(T_, chunk);
    const int ngr = cdiv(nch, kBY);
    const int b = by / ngr;
    const int ci = (by - b * ngr) * kBY + threadIdx.y;
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
      if constexpr (sizeof(T) == 2) {
        // bf16: rows and taps stay packed (two channels a word) and every product is a
        // mixed fma.rn.f32.bf16 (exact product, one rounding: the same results as widening
        // first), which halves the registers the windows take and needs no unpacking
        constexpr int NW = V / 2;
        using RT = typename P::raw_t;
        auto words = [](const RT &r, uint32_t (&o)[NW]) {
            const uint32_t *q = reinterpret_cast<const uint32_t *>(&r);
#pragma unroll
            for (int j = 0; j < NW; ++j) o[j] = q[j];
        };
        uint32_t fw[W][NW];          // (w[c0+2j, k], w[c0+2j+1, k])
        {
            const uint16_t *wr = reinterpret_cast<const uint16_t *>(ws);
#pragma unroll
            for (int j = 0; j < NW; ++j)
#pragma unroll
                for (int k = 0; k < W; ++k)
                    fw[k][j] = (uint32_t)__ldg(wr + (size_t)(c0 + 2 * j) * W + k) |
                               ((uint32_t)__ldg(wr + (size_t)(c0 + 2 * j + 1) * W + k) << 16);
        }
        constexpr bool kRing = kU % W == 0;
        const bool ring = kRing && (t1 - t0) % W == 0;
        uint32_t xw[W][NW], dyw[W][NW];
#pragma unroll
        for (int k = 1; k < W; ++k) {
            uint32_t r[NW];
            if (t0 - k >= 0) words(P::load(x + off + (size_t)(t0 - k) * D), r);
            else
#pragma unroll
                for (int j = 0; j < NW; ++j) r[j] = 0u;
            const int sk = (kRing && ring) ? W - k : k;      // slot of row t0-k
#pragma unroll
            for (int j = 0; j < NW; ++j) {
                xw[sk][j] = r[j];
                dyw[sk][j] = 0u;        // rows before t0 feed no dx row of this chunk
            }
        }
        auto step = [&](int t, bool in_chunk, auto sl) {
            if (in_chunk) {
#pragma unroll
                for (int k = 0; k < W; ++k)
#pragma unroll
                    for (int j = 0; j < NW; ++j) {
                        acc[k][2 * j] = fma_bf16_lo(dyw[sl(0)][j], xw[sl(k)][j], acc[k][2 * j]);
                        acc[k][2 * j + 1] = fma_bf16_hi(dyw[sl(0)][j], xw[sl(k)][j], acc[k][2 * j + 1]);
                    }
            }
            const int s = t - (W - 1);
            if (s >= t0) {
                float o[V];
#pragma unroll
                for (int j = 0; j < NW; ++j) {
                    float a0 = bf16_lo(dyw[sl(W - 1)][j]), a1 = bf16_hi(dyw[sl(W - 1)][j]);
#pragma unroll
                    for (int k = 0; k < W; ++k) {
                        a0 = fma_bf16_lo(fw[k][j], dyw[sl(W - 1 - k)][j], a0);
                        a1 = fma_bf16_hi(fw[k][j], dyw[sl(W - 1 - k)][j], a1);
                    }
                    o[2 * j] = a0;
                    o[2 * j + 1] = a1;
                }
                P::store(dx + off + (size_t)s * D, o);
            }
        };
        auto shift = [&]() {
#pragma unroll
            for (int k = W - 1; k >= 1; --k)
#pragma unroll
                for (int j = 0; j < NW; ++j) {
                    dyw[k][j] = dyw[k - 1][j];
                    xw[k][j] = xw[k - 1][j];
                }
        };
        const Staging<P::BYTES, 2, kU, kBX * kBY> stg((uint32_t)__cvta_generic_to_shared(stg_raw),
                                                  (int)(threadIdx.y * kBX + threadIdx.x));
        auto issue = [&](int tb, int stage) {
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const bool ok = tb + u < t1;
                const size_t r = (size_t)(ok ? tb + u : t0) * D;
                cp_async<P::BYTES>(stg.at(stage, 0, u), x + off + r, ok);
                cp_async<P::BYTES>(stg.at(stage, 1, u), dy + off + r, ok);
            }
            cp_commit();
        };
        const int nb = cdiv(t1 - t0, kU);
        issue(t0, 0);
        for (int bi = 0; bi < nb; ++bi) {
            const int tb = t0 + bi * kU, stage = bi & 1;
            if (bi + 1 < nb) issue(tb + kU, stage ^ 1);
            else cp_commit();
            cp_wait<1>();
            if (kRing && ring) {
#pragma unroll
                for (int u = 0; u < kU; ++u) {
                    if (tb + u >= t1) break;
                    const int s0 = u % W;
                    words(lds_raw<RT>(stg.at(stage, 0, u)), xw[s0]);
                    words(lds_raw<RT>(stg.at(stage, 1, u)), dyw[s0]);
                    step(tb + u, true, [&](int k) { return (u - k + W) % W; });
                }
            } else {
#pragma unroll
                for (int u = 0; u < kU; ++u) {
                    if (tb + u >= t1) break;
                    words(lds_raw<RT>(stg.at(stage, 0, u)), xw[0]);
                    words(lds_raw<RT>(stg.at(stage, 1, u)), dyw[0]);
                    step(tb + u, true, [](int k) { return k; });
                    shift();
                }
            }
        }
        cp_wait<0>();
        // rows t1-W+1 .. t1-1 need dy rows t1 .. t1+W-2 (zero past the sequence end)
#pragma unroll
        for (int e = 0; e < W - 1; ++e) {
            const int t = t1 + e;
            uint32_t r[NW];
            if (t < T_) words(P::load(dy + off + (size_t)t * D), r);
            else
#pragma unroll
                for (int j = 0; j < NW; ++j) r[j] = 0u;
            if (kRing && ring) {       // row t1+e is in slot e % W
#pragma unroll
                for (int j = 0; j < NW; ++j) dyw[e % W][j] = r[j];
                step(t, false, [&](int k) { return (e - k + W) % W; });
            } else {
#pragma unroll
                for (int j = 0; j < NW; ++j) dyw[0][j] = r[j];
                step(t, false, [](int k) { return k; });
                shift();
            }
        }
      } else {
        float f[W][V];
#pragma unroll
        for (int i = 0; i < V; ++i)
#pragma unroll
            for (int k = 0; k < W; ++k) f[k][i] = to_f(__ldg(ws + (size_t)(c0 + i) * W + k));
        // The windows of x and dy rows: a ring (row r in slot (r - t0) % W, a constant in
        // every unrolled step, no copies) when a batch is a whole number of windows and
        // the chunk is too; else shifted down one slot per token (xw[k] = row t-k).
        constexpr bool kRing = kU % W == 0;
        const bool ring = kRing && (t1 - t0) % W == 0;
        float xw[W][V], dyw[W][V];
#pragma unroll
        for (int k = 1; k < W; ++k) {
            float r[V];
            if (t0 - k >= 0) P::unpack(P::load(x + off + (size_t)(t0 - k) * D), r);
            else
#pragma unroll
                for (int i = 0; i < V; ++i) r[i] = 0.f;
            const int sk = (kRing && ring) ? W - k : k;      // slot of row t0-k
#pragma unroll
            for (int i = 0; i < V; ++i) {
                xw[sk][i] = r[i];
                dyw[sk][i] = 0.f;       // rows before t0 feed no dx row of this chunk
            }
        }
        // one token t, its x and dy rows already in slot sl(0); sl(k) is the slot of row t-k
        auto step = [&](int t, bool in_chunk, auto sl) {
            if (in_chunk) {
#pragma unroll
                for (int k = 0; k < W; ++k)
#pragma unroll
                    for (int i = 0; i < V; ++i) acc[k][i] = fmaf(dyw[sl(0)][i], xw[sl(k)][i], acc[k][i]);
            }
            const int s = t - (W - 1);
            if (s >= t0) {
                float o[V];
#pragma unroll
                for (int i = 0; i < V; ++i) {
                    float a = dyw[sl(W - 1)][i];
#pragma unroll
                    for (int k = 0; k < W; ++k) a = fmaf(f[k][i], dyw[sl(W - 1 - k)][i], a);
                    o[i] = a;
                }
                P::store(dx + off + (size_t)s * D, o);
            }
        };
        auto shift = [&]() {
#pragma unroll
            for (int k = W - 1; k >= 1; --k)
#pragma unroll
                for (int i = 0; i < V; ++i) {
                    dyw[k][i] = dyw[k - 1][i];
                    xw[k][i] = xw[k - 1][i];
                }
        };
        const Staging<P::BYTES, 2, kU, kBX * kBY> stg((uint32_t)__cvta_generic_to_shared(stg_raw),
                                                  (int)(threadIdx.y * kBX + threadIdx.x));
        auto issue = [&](int tb, int stage) {
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const bool ok = tb + u < t1;
                const size_t r = (size_t)(ok ? tb + u : t0) * D;
                cp_async<P::BYTES>(stg.at(stage, 0, u), x + off + r, ok);
                cp_async<P::BYTES>(stg.at(stage, 1, u), dy + off + r, ok);
            }
            cp_commit();
        };
        const int nb = cdiv(t1 - t0, kU);
        issue(t0, 0);
        for (int bi = 0; bi < nb; ++bi) {
            const int tb = t0 + bi * kU, stage = bi & 1;
            if (bi + 1 < nb) issue(tb + kU, stage ^ 1);
            else cp_commit();
            cp_wait<1>();
            if (kRing && ring) {
#pragma unroll
                for (int u = 0; u < kU; ++u) {
                    if (tb + u >= t1) break;
                    const int s0 = u % W;
                    P::unpack(lds_raw<typename P::raw_t>(stg.at(stage, 0, u)), xw[s0]);
                    P::unpack(lds_raw<typename P::raw_t>(stg.at(stage, 1, u)), dyw[s0]);
                    step(tb + u, true, [&](int k) { return (u - k + W) % W; });
                }
            } else {
#pragma unroll
                for (int u = 0; u < kU; ++u) {
                    if (tb + u >= t1) break;
                    P::unpack(lds_raw<typename P::raw_t>(stg.at(stage, 0, u)), xw[0]);
                    P::unpack(lds_raw<typename P::raw_t>(stg.at(stage, 1, u)), dyw[0]);
                    step(tb + u, true, [](int k) { return k; });
                    shift();
                }
            }
        }
        cp_wait<0>();
        // rows t1-W+1 .. t1-1 need dy rows t1 .. t1+W-2 (zero past the sequence end)
#pragma unroll
        for (int e = 0; e < W - 1; ++e) {
            const int t = t1 + e;
            float r[V];
            if (t < T_) P::unpack(P::load(dy + off + (size_t)t * D), r);
            else
#pragma unroll
                for (int i = 0; i < V; ++i) r[i] = 0.f;
            if (kRing && ring) {       // row t1+e is in slot e % W
#pragma unroll
                for (int i = 0; i < V; ++i) dyw[e % W][i] = r[i];
                step(t, false, [&](int k) { return (e - k + W) % W; });
            } else {
#pragma unroll
                for (int i = 0; i < V; ++i) dyw[0][i] = r[i];
                step(t, false, [](int k) { return k; });
                shift();
            }
        }
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
                part[((size_t)by * D + c0 + i) * W + k] = s;
            }
        }
        __syncthreads();
    }
}

template <typename T, int W>
__global__ void __launch_bounds__(kBX * kBY)
k_static_bwd(const T *__restrict__ x, const T *__restrict__ ws, const T *__restrict__ dy, T *__restrict__ dx,
             float *__restrict__ part, int B, int T_, int D, int chunk) {
    // persistent: work item = (kBX channel vectors, kBY chunks of one sequence)
    constexpr int V = Lanes<T, W>::V;
    const int nbx = cdiv(D / V, kBX);
    const int nitems = nbx * dw_partials(B, T_);
    for (int item = blockIdx.x; item < nitems; item += gridDim.x)
        static_bwd_item<T, W>(x, ws, dy, dx, part, B, T_, D, chunk, item % nbx, item / nbx);
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


// Blocks of `kern` that fit on the device at once (at least one per SM).
template <typename K>
int resident_blocks(K kern, int threads, int smem) {
    int dev = 0, nsm = 148, per = 1;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, kern, threads, smem) != cudaSuccess || per < 1) per = 1;
    return nsm * per;
}

template <typename T>
bool launch_dyn_bwd_T(const void *x, const void *w, const void *dy, void *dx, float *dw, int B, int T_, int D,
                      int G, int W, cudaStream_t s) {
    const T *xp = (const T *)x, *wp = (const T *)w, *gp = (const T *)dy;
    T *op = (T *)dx;
    constexpr int kRows = 64;   // tokens per chunk
    switch (W) {
#define DSC_CASE(WW)                                                                                   \
    case WW: {                                                                                         \
        constexpr int V = Lanes<T, WW>::V;                                                             \
        constexpr int TB = WW * (int)sizeof(T);                                                        \
        if constexpr (TB == 4 || TB == 8 || TB == 16) {                                                \
            if (G % V != 0 || G / V > 32 || ((G / V) & (G / V - 1)) != 0) return false;                \
            constexpr int SB = Pack<T, V>::BYTES > TB ? Pack<T, V>::BYTES : TB;                        \
            const int smem = 256 * Staging<SB, 3, Batch<SB>::KU>::bytes_per_thread();                  \
            auto kern = k_dyn_bwd<T, WW>;                                                              \
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);             \
            const long long items = (long long)cdiv(D / V, 256) * B * cdiv(T_, kRows);                 \
            const int grid = (int)std::min<long long>(items, (long long)resident_blocks(kern, 256, smem)); \
            kern<<<grid, 256, smem, s>>>(xp, wp, gp, op, dw, B, T_, D, G, kRows);                       \
            return true;                                                                               \
        } else {                                                                                       \
            return false;                                                                              \
        }                                                                                              \
    }
        DSC_CASE(1) DSC_CASE(2) DSC_CASE(3) DSC_CASE(4) DSC_CASE(5) DSC_CASE(6) DSC_CASE(7) DSC_CASE(8)
#undef DSC_CASE
    }
    return false;
}

template <typename T, int W, bool STATIC>
void launch_fwd_k(int nitems, const T *x, const T *w, T *y, int B, int T_, int D, int G, int chunk,
                  cudaStream_t s) {
    constexpr int V = Lanes<T, W>::V;
    constexpr int PB = V * (int)sizeof(T);
    constexpr int TB = W * (int)sizeof(T);
    constexpr bool kTapVec = !STATIC && (TB == 4 || TB == 8 || TB == 16);
    constexpr int SB = PB > TB || !kTapVec ? PB : TB;
    constexpr int smem = 256 * Staging<SB, kTapVec ? 2 : 1, Batch<SB>::KU>::bytes_per_thread();
    auto kern = k_stream_fwd<T, W, STATIC>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    // one work item per block: short-lived blocks overlap each other's first loads
    kern<<<nitems, 256, smem, s>>>(x, w, y, B, T_, D, G, chunk);
}

template <typename T, bool STATIC>
void launch_stream_fwd_T(const void *x, const void *w, void *y, int B, int T_, int D, int G, int W,
                         cudaStream_t s) {
    const int chunk = chunk_fwd(T_, W);
    const T *xp = (const T *)x;
    const T *wp = (const T *)w;
    T *yp = (T *)y;
    switch (W) {
#define DSC_CASE(WW)                                                                                  \
    case WW: {                                                                                        \
        constexpr int V = Lanes<T, WW>::V;                                                            \
        launch_fwd_k<T, WW, STATIC>(cdiv(D / V, 256) * B * cdiv(T_, chunk), xp, wp, yp, B, T_, D, G,  \
                                    chunk, s);                                                        \
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
        constexpr int SB = V * (int)sizeof(T);                                                        \
        const int smem = kBX * kBY * Staging<SB, 2, Batch<SB>::KU, kBX * kBY>::bytes_per_thread();    \
        auto kern = k_static_bwd<T, WW>;                                                              \
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);                \
        const int grid = std::min(cdiv(D / V, kBX) * P, resident_blocks(kern, kBX * kBY, smem));      \
        kern<<<grid, dim3(kBX, kBY), smem, s>>>(xp, wp, gp, op, part, B, T_, D, chunk);               \
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

int static_dw_partials(int B, int T) { return dw_partials(B, T); }

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

bool launch_dyn_bwd(const void *x, const void *w, const void *dy, void *dx, float *dw, int B, int T, int D, int G,
                    int W, bool bf16_, cudaStream_t s) {
    return bf16_ ? launch_dyn_bwd_T<bf16>(x, w, dy, dx, dw, B, T, D, G, W, s)
                 : launch_dyn_bwd_T<float>(x, w, dy, dx, dw, B, T, D, G, W, s);
}

void launch_static_bwd(const void *x, const void *w, const void *dy, void *dx, float *part, float *dw, int B,
                       int T, int D, int W, bool bf16_, cudaStream_t s) {
    if (bf16_) launch_static_bwd_T<bf16>(x, w, dy, dx, part, dw, B, T, D, W, s);
    else launch_static_bwd_T<float>(x, w, dy, dx, part, dw, B, T, D, W, s);
}

}  // namespace dsc
