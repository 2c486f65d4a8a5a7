// Tensor-core (tcgen05 / TMEM / TMA) kernels for the fused low-rank causal dynamic
// short convolution on sm_100a.
//
// "Convolucoes Curtas Dinamicas Melhoram Transformers", Implementacao de Treinamento
// Eficiente: the fused low-rank kernel reads z and U, forms the filters zU on chip and
// applies the convolution at once, so the full filter tensor never reaches HBM.
//
// Forward, per CTA work tile = 128 tokens of one sequence x one 64-channel slice:
//   w[t, j] = sum_r z[t, r] U[r, c0*W/G + j]      tcgen05.mma, M=128 (tokens), K=R,
//                                                 N = (64/G)*W columns, fp32 in TMEM
//   y[t, c] = x[t, c] + sum_k w[t, g(c)W+k] x[t-k, c]
// The x tile (plus its W-1 row causal halo; TMA fills rows before t=0 with zeros),
// the z tile and the U slice arrive by TMA; y leaves through shared memory by TMA.
//
// Warp roles (persistent CTAs, one per SM, tiles in token-major round-robin order):
//   warp 0  TMA producer of the x tiles, into an x ring that the epilogue releases
//   warp 18 (after the epilogue warps) TMA producer of the MMA operands of a tile (z tile,
//           U slice), into a 2-deep operand ring that the MMA releases as soon as its
//           MMAs complete.  The two producers are independent, so the x loads run several
//           tiles ahead of the epilogue, which both epilogue sets need (each holds one x
//           stage while it works), whatever the operand ring does.
//   warp 1  TMEM allocator and MMA issuer (one elected lane), double-buffered accumulator
//   warps 2-17  two epilogue sets of 8 warps taking alternating tiles: warp w reads TMEM
//              lanes 32*(w%4).. (its 32 tokens) and handles 32 channels (half the slice);
//              one token row per thread.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstdio>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"

namespace dsc {
namespace tc {

__device__ unsigned int g_fault = 0;

// Waiting warps sleep on their mbarrier (up to this many ns per try) rather than poll:
// the two epilogue sets spend much of each tile waiting, and their polling takes issue
// slots from the set that is computing (about 4% of the forward's time).
constexpr unsigned kWaitHint = 2000;

// Build-time tuning constants of the forward kernel.
#ifndef DSC_FWD_SETS
#define DSC_FWD_SETS 2         // epilogue warp sets working on alternating tiles (1 or 2)
#endif
#ifndef DSC_FWD_CHPAIR
#define DSC_FWD_CHPAIR 1       // groups of 4+ channels: fp32x2 FMAs over channel pairs
#endif
#ifndef DSC_FWD_F32X2
#define DSC_FWD_F32X2 2        // pair taps with packed fp32x2 FMAs: 1 always, 0 never, 2 for W <= 4
#endif
#ifndef DSC_X_L2_PROMO
#define DSC_X_L2_PROMO 128     // L2 promotion of the x tile loads (128 or 256 bytes)
#endif

constexpr int kTt = 128;          // tokens per tile (MMA M)
constexpr int kDt = 64;           // channels per slice

struct FwdParams {
    int B, T, D, G, R;
    int n_slices;             // D / 64
    int tiles_per_seq;
    int n_tiles;              // tiles in token-major order: i = token_tile * n_slices + slice
    int slice_cols;           // (64/G)*W
    int n_pad;                // slice_cols rounded up to 16
    int u_boxes;              // ceil(n_pad / 64) TMA boxes of 64 columns
    int bufcols, nbuf, tmem_cols;
    int stages, nwg;          // x ring depth; nwg: epilogue warp sets (1 or 2)
    int op_stages;            // operand (z, U) ring depth
    uint32_t x_stage_tx, x_stage_bytes, z_stage_bytes, u_bytes, y_buf_bytes;
    uint32_t op_bytes;        // one operand stage: z tile and U slice
    uint32_t off_x, off_op, off_y, off_bar;   // ring bases
    uint32_t off_z, off_u;    // within an operand stage
    uint32_t z_layout;        // swizzle of the z tile (32/64/128-byte rows)
    const float *cs;          // RoPE table [T][dh/2][2] (cos, sin), or null
    int dh, n_rot;            // RoPE head size; channels [0, n_rot) rotated (0: none)
    WaitTest wt;
};

// Decode step (one new token per sequence): the kernel's token rows are the B sequences
// (a "sequence" of B rows, z_t [B, R] as its z), and an x stage holds, per sequence, x_t
// and its rolling window state [B, W-1, D] instead of a token tile and its halo.  The
// window is read through a view with the sequence as the middle dimension (dims
// {D, B, W-1}), so that one box lands in shared memory as [window row][128 sequences]
// [64 channels] and rows 1.. of it are again one box: `load` (all W-1 rows), `shift`
// (W-2 rows, stage rows 1.. to window rows 0..) and `push` (x_t to the newest row).
struct DecMaps {
    CUtensorMap load, shift, push;
};
constexpr uint32_t kDecRow = 128 * 128;       // one [128 sequences][64 channels] bf16 region

// Barrier slots in shared memory (8 bytes each).
constexpr int kMaxXStages = 8;
constexpr int kOpStages = 2;

struct Bars {
    uint32_t base;
    __device__ uint32_t full(int s) const { return base + 8 * s; }
    __device__ uint32_t empty(int s) const { return base + 8 * (kMaxXStages + s); }
    __device__ uint32_t ofull(int o) const { return base + 8 * (2 * kMaxXStages + o); }
    __device__ uint32_t oempty(int o) const { return base + 8 * (2 * kMaxXStages + kOpStages + o); }
    __device__ uint32_t accf(int a) const { return base + 8 * (2 * kMaxXStages + 2 * kOpStages + a); }
    __device__ uint32_t acce(int a) const { return base + 8 * (2 * kMaxXStages + 2 * kOpStages + 2 + a); }
    __device__ uint32_t done() const { return base + 8 * (2 * kMaxXStages + 2 * kOpStages + 4); }
};
constexpr uint32_t kBarBytes = 8 * (2 * kMaxXStages + 2 * kOpStages + 5);

__device__ __forceinline__ void unpack8(const uint4 &u, float (&v)[8]) {
    v[0] = bf16_lo(u.x); v[1] = bf16_hi(u.x);
    v[2] = bf16_lo(u.y); v[3] = bf16_hi(u.y);
    v[4] = bf16_lo(u.z); v[5] = bf16_hi(u.z);
    v[6] = bf16_lo(u.w); v[7] = bf16_hi(u.w);
}

__host__ __device__ constexpr int pow2_divisor(int n, int cap) {
    int p = 1;
    while (p * 2 <= cap && n % (p * 2) == 0) p *= 2;
    return p;
}

// Filter taps of one 8-channel chunk, read from TMEM:
//   GC <= 8: 8/GC groups x W taps in U's column order (column gl*W + k), a contiguous
//            block of NCOL columns loaded in aligned pieces of PIECE columns;
//   GC == 16 (any G >= 16): one group, W columns.
template <int W, int GC>
struct Taps {
    static constexpr int NCOL = GC <= 8 ? (8 / GC) * W : W;
    static constexpr int PIECE = GC <= 8 ? pow2_divisor(NCOL, 64) : 1;
};

// Epilogue: each set of 8 warps covers one whole tile (warp = 32 token rows x 32
// channels); with two sets, consecutive tiles (the two TMEM accumulator buffers) are
// processed concurrently.  Two sets need the chunk's taps to fit in 32 registers, and
// at least two x stages: a set waits for phase n of its stage's barrier before the
// phases in between have completed, which an mbarrier's parity cannot tell apart when
// both sets share one stage.  The decode step keeps one set (its stages are W x 16 KB).
template <int W, int GC, bool DEC = false>
struct EpiShape {
    static constexpr int SETS = (!DEC && Taps<W, GC>::NCOL <= 32 && DSC_FWD_SETS >= 2) ? 2 : 1;
    static constexpr int WARPS = 8 * SETS;
    static constexpr int OPWARP = 2 + WARPS;       // the operand (z, U) producer
    static constexpr int THREADS = 32 * (3 + WARPS);
    static constexpr int CPW = 32;                 // channels per epilogue warp
    static constexpr int CHUNKS = CPW / 8;
    static constexpr int YBUF = 32 * CPW * 2;      // one warp's y staging: 32 rows x 32 bf16
};

// y[t,c] = x[t,c] + sum_k w[t, g(c), k] x[t-k, c] for the 8 channels of one chunk.
template <int W, int GC>
__device__ __forceinline__ void conv_chunk(const uint32_t *wr, const uint4 (&xu)[W], float (&out)[8]) {
    float xv[W][8];
#pragma unroll
    for (int k = 0; k < W; ++k) unpack8(xu[k], xv[k]);
    if constexpr (GC >= 4 && DSC_FWD_CHPAIR) {
        // a group spans at least 4 channels: channel pairs (2m, 2m+1) share its taps, so
        // packed fp32x2 FMAs take the two channels at once (each tap duplicated once per
        // group; the same fmaf sequence per channel as the scalar form)
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const int gl = GC <= 8 ? (2 * m) / GC : 0;
            const uint32_t *wg = wr + gl * W;
            uint64_t acc = f2pack(xv[0][2 * m], xv[0][2 * m + 1]);
#pragma unroll
            for (int k = 0; k < W; ++k) {
                const float wk = __uint_as_float(wg[k]);
                acc = f2fma(f2pack(wk, wk), f2pack(xv[k][2 * m], xv[k][2 * m + 1]), acc);
            }
            f2unpack(acc, out[2 * m], out[2 * m + 1]);
        }
    } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const int gl = GC <= 8 ? e / GC : 0;
            const uint32_t *wg = wr + gl * W;
            // measured: the packed form is faster with 4 taps (lowrank_qkv 0.095 -> 0.091 ms)
            // and slower with 8 (lowrank_mlp 0.145 -> 0.157 ms)
            constexpr bool kPair = DSC_FWD_F32X2 == 1 || (DSC_FWD_F32X2 == 2 && W <= 4);
            if constexpr (kPair && W >= 2) {
                // taps in pairs with packed fp32x2 FMAs (two partial sums, added at the end)
                uint64_t acc = f2pack(xv[0][e], 0.f);
#pragma unroll
                for (int k = 0; k + 1 < W; k += 2)
                    acc = f2fma(f2pack(__uint_as_float(wg[k]), __uint_as_float(wg[k + 1])),
                                f2pack(xv[k][e], xv[k + 1][e]), acc);
                float a0, a1;
                f2unpack(acc, a0, a1);
                if (W & 1) a0 = fmaf(__uint_as_float(wg[W - 1]), xv[W - 1][e], a0);
                out[e] = a0 + a1;
            } else {
                float acc = xv[0][e];
#pragma unroll
                for (int k = 0; k < W; ++k) acc = fmaf(__uint_as_float(wg[k]), xv[k][e], acc);
                out[e] = acc;
            }
        }
    }
}

// The whole kernel, for the forward (DEC false: tiles of 128 tokens of one sequence) and
// the decode step (DEC true: tiles of 128 sequences, one token each).  The maps are the
// kernels' grid-constant parameters.
template <int W, int GC, bool ROPE, bool DEC>
__device__ __forceinline__ void fwd_tiles(const CUtensorMap &tm_x, const CUtensorMap &tm_z, const CUtensorMap &tm_u,
                                          const CUtensorMap &tm_y, const DecMaps *dm, const FwdParams &p) {
    using ES = EpiShape<W, GC, DEC>;
    using TP = Taps<W, GC>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const uint32_t sb = smem_u32(smem);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const Bars bar{sb + p.off_bar};
    uint32_t *tmem_holder = (uint32_t *)(smem + p.off_bar + kBarBytes);
    volatile int *abort = (volatile int *)(smem + p.off_bar + kBarBytes + 8);

    if (threadIdx.x == 0) {
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(bar.full(s), 1);
            mbar_init(bar.empty(s), 8);
        }
        for (int o = 0; o < p.op_stages; ++o) {
            mbar_init(bar.ofull(o), 1);
            mbar_init(bar.oempty(o), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(bar.accf(a), 1);
            mbar_init(bar.acce(a), 8);
        }
        mbar_init(bar.done(), 1);
        *abort = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch(&tm_x);
        tma_prefetch(&tm_z);
        tma_prefetch(&tm_u);
        tma_prefetch(&tm_y);
        if (DEC && W > 1) {
            tma_prefetch(&dm->load);
            if (W > 2) tma_prefetch(&dm->shift);
            tma_prefetch(&dm->push);
        }
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_holder), p.tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    const int S = p.stages;

    if (warp == 0) {
        // ---------------------------------------------------------- TMA producer
        if (lane == 0) {
            int it = 0;
            for (int i = blockIdx.x; i < p.n_tiles; i += gridDim.x, ++it) {
                const int slice = i % p.n_slices, tl_ = i / p.n_slices;
                const int b = tl_ / p.tiles_per_seq, t0 = (tl_ % p.tiles_per_seq) * kTt;
                const int s = it % S, n = it / S;
                if (!mbar_wait<kWaitHint>(bar.empty(s), (n & 1) ^ 1, abort, 2u, &g_fault, p.wt.wait_ns)) break;
                if (it == 0 && (int)blockIdx.x == p.wt.withhold_cta) continue;   // test hook: no loads
                const uint32_t xs = sb + p.off_x + s * p.x_stage_bytes;
                if constexpr (DEC) {
                    // x_t of the tile's sequences, then their windows; the stage's shift
                    // stores of the previous round must have read it first
                    if (W > 1) bulk_wait_read<0>();
                    mbar_arrive_expect_tx(bar.full(s), p.x_stage_tx);
                    tma_load_3d(xs, &tm_x, bar.full(s), slice * kDt, t0, b);
                    if (W > 1) {
                        tma_load_3d(xs + kDecRow, &dm->load, bar.full(s), slice * kDt, t0, 0);
                        // once both have landed the window moves on in global memory: rows
                        // 1..W-2 to rows 0..W-3 and x_t into row W-2 (only this tile's
                        // sequences and channels, which no other tile reads)
                        if (!mbar_wait<kWaitHint>(bar.full(s), n & 1, abort, 2u, &g_fault, p.wt.wait_ns)) break;
                        if (W > 2) tma_store_3d(&dm->shift, xs + 2 * kDecRow, slice * kDt, t0, 0);
                        tma_store_3d(&dm->push, xs, slice * kDt, t0, W - 2);
                        bulk_commit();
                    }
                } else {
                    mbar_arrive_expect_tx(bar.full(s), p.x_stage_tx);
                    tma_load_3d(xs, &tm_x, bar.full(s), slice * kDt, t0 - (W - 1), b);
                }
            }
            // Let every load this warp issued land before the CTA can exit.
            const int issued = it;
            for (int s = 0; s < S && s < issued; ++s) {
                const int last = issued - 1 - ((issued - 1 - s) % S);   // last tile using stage s
                mbar_drain(bar.full(s), (last / S) & 1, p.wt.wait_ns);
            }
            if (DEC) bulk_wait_all();    // the window stores are complete
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        // The whole warp waits; one elected lane then issues a tile's tcgen05 instructions
        // in a row, descriptors advancing by adds to their start-address field.
        const int nchunks = (p.n_pad + 255) / 256;
        const uint32_t ubox = (uint32_t)(p.R * 128);
        const int ksteps = p.R / 16;
        const uint64_t t_z = desc_tmpl(16, 8u * p.R * 2u, p.z_layout);   // z tile, K-major
        const uint64_t t_u = desc_tmpl(ubox, 1024, kSw128);              // U slice, MN-major
        const uint32_t i_full = idesc_bf16(128, 256, false, true);
        const uint32_t i_last = idesc_bf16(128, p.n_pad - 256 * (nchunks - 1), false, true);
        int it = 0, a = 0, m = 0;    // accumulator a of round m, advanced by increments
        for (int i = blockIdx.x; i < p.n_tiles; i += gridDim.x, ++it) {
            const int o = it % kOpStages, on = it / kOpStages;
            if (!warp_wait<kWaitHint>(bar.ofull(o), on & 1, abort, 8u, &g_fault, p.wt.wait_ns)) break;
            if (!warp_wait<kWaitHint>(bar.acce(a), (m & 1) ^ 1, abort, 16u, &g_fault, p.wt.wait_ns)) break;
            tc_fence_after();
            const uint32_t d = tmem + a * p.bufcols;
            const uint32_t za = sb + p.off_op + o * p.op_bytes + p.off_z;
            const uint32_t ua = sb + p.off_op + o * p.op_bytes + p.off_u;
            if (elect_one()) {      // one lane issues the tile's MMAs and commits
                for (int nc = 0; nc < nchunks; ++nc) {
                    const uint32_t idesc = nc + 1 < nchunks ? i_full : i_last;
                    uint64_t dz = desc_at(t_z, za), du = desc_at(t_u, ua + nc * 4 * ubox);
                    for (int kk = 0; kk < ksteps; ++kk) {
                        mma_bf16_ss(d + 256 * nc, dz, du, idesc, kk > 0 ? 1u : 0u);
                        dz += 32u >> 4;
                        du += 2048u >> 4;
                    }
                }
                mma_commit(bar.accf(a));
                mma_commit(bar.oempty(o));
            }
            __syncwarp();
            if (++a == p.nbuf) { a = 0; ++m; }
        }
        if (elect_one()) mma_commit(bar.done());
        __syncwarp();
    } else if (warp == ES::OPWARP) {
        // ---------------------------------------------------------- TMA producer: operands
        if (lane == 0) {
            int it = 0;
            for (int i = blockIdx.x; i < p.n_tiles; i += gridDim.x, ++it) {
                const int slice = i % p.n_slices, tl_ = i / p.n_slices;
                const int b = tl_ / p.tiles_per_seq, t0 = (tl_ % p.tiles_per_seq) * kTt;
                const int o = it % kOpStages, on = it / kOpStages;
                if (!mbar_wait<kWaitHint>(bar.oempty(o), (on & 1) ^ 1, abort, 2u, &g_fault, p.wt.wait_ns)) break;
                if (it == 0 && (int)blockIdx.x == p.wt.withhold_cta) continue;   // test hook: no loads
                const uint32_t os = sb + p.off_op + o * p.op_bytes;
                mbar_arrive_expect_tx(bar.ofull(o), p.z_stage_bytes + p.u_bytes);
                tma_load_3d(os + p.off_z, &tm_z, bar.ofull(o), 0, t0, b);
                for (int bx = 0; bx < p.u_boxes; ++bx)
                    tma_load_2d(os + p.off_u + bx * (uint32_t)(p.R * 128), &tm_u, bar.ofull(o),
                                slice * p.slice_cols + 64 * bx, 0);
            }
            const int issued = it;
            for (int o = 0; o < p.op_stages && o < issued; ++o) {
                const int last = issued - 1 - ((issued - 1 - o) % p.op_stages);
                mbar_drain(bar.ofull(o), (last / p.op_stages) & 1, p.wt.wait_ns);
            }
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------- epilogue
        const int ew = warp - 2;
        const int set = ew >> 3;             // tiles it with it % SETS == set
        const int q = warp & 3;              // TMEM lane quarter == token rows 32q..32q+31
        const int h = (ew >> 2) & 1;         // channel half of the slice
        const int row = 32 * q + lane;       // token row in the tile
        // y staging: row `lane` of this warp's buffer, 64-byte swizzle (16-byte chunk ^ (lane/2)%4)
        const uint32_t ystage = sb + p.off_y + (uint32_t)ew * 2 * ES::YBUF;
        const uint32_t yrow = (ystage + lane * 64) ^ ((uint32_t)((lane >> 1) & 3) << 4);
        // x stage: the thread's rows r_k = row + W-1-k (decode: x_t in region 0, window
        // row W-1-k in region W-k, a region being 128 rows); a row is 128 bytes with
        // 128-byte swizzle (16-byte chunk ^ r%8).  Rows are 128-byte aligned, so the
        // swizzled address of chunk c is (row address ^ ((r%8) << 4)) ^ (c << 4).
        uint32_t xrow[W];
#pragma unroll
        for (int k = 0; k < W; ++k) {
            const uint32_t r = DEC ? (uint32_t)((k == 0 ? 0 : W - k) * kTt + row) : (uint32_t)(row + (W - 1) - k);
            xrow[k] = (r * 128u) ^ ((r & 7u) << 4) ^ ((uint32_t)(4 * h) << 4);
        }
        int yc = 0;
        const int it0 = set;
        int i = blockIdx.x + set * gridDim.x;
        // this set's position, advanced by increments: slice and token tile (tlin; its
        // sequence b and tile tt within it), x stage s of round n, accumulator a of round m
        int slice = i % p.n_slices, tlin = i / p.n_slices;
        int b = tlin / p.tiles_per_seq, tt = tlin - b * p.tiles_per_seq;
        int s = it0 % S, n = it0 / S, a = it0 % p.nbuf, m = it0 / p.nbuf;
        const int step = ES::SETS * gridDim.x;
        const int dslice = step % p.n_slices, dtl = step / p.n_slices;
        for (; i < p.n_tiles; i += step) {
            const int t0 = tt * kTt;
            // RoPE (when on): channel pairs (2i, 2i+1) of the first n_rot channels rotated by
            // the angle of pair i = (c mod dh) / 2 at this row's position in its sequence.
            // A chunk's 4 (cos, sin) pairs are read one chunk ahead (the first before the
            // waits); the table is pair-major, so a warp's 32 rows read 256 contiguous bytes.
            const int c_warp = slice * kDt + ES::CPW * h;
            const bool rot_row = ROPE && t0 + row < p.T;
            float2 csn[4];
            auto load_cs = [&](int cq) {
                const int c8 = c_warp + 8 * cq;
                if (rot_row && c8 < p.n_rot) {
                    const float2 *src = reinterpret_cast<const float2 *>(p.cs) +
                                        (size_t)((c8 % p.dh) / 2) * p.T + (t0 + row);
#pragma unroll
                    for (int m2 = 0; m2 < 4; ++m2) csn[m2] = __ldg(src + (size_t)m2 * p.T);
                }
            };
            if (ROPE) load_cs(0);
            if (!warp_wait<kWaitHint>(bar.full(s), n & 1, abort, 32u, &g_fault, p.wt.wait_ns)) break;
            if (!warp_wait<kWaitHint>(bar.accf(a), m & 1, abort, 64u, &g_fault, p.wt.wait_ns)) break;
            tc_fence_after();
            const int yb = yc & 1;
            if (lane == 0) bulk_wait_read<1>();
            __syncwarp();
            const uint32_t xs = sb + p.off_x + s * p.x_stage_bytes;
            const uint32_t tl = tmem + ((uint32_t)(32 * q) << 16) + a * p.bufcols;
            const uint32_t yw = yrow + yb * ES::YBUF;
            uint32_t wr[2][TP::NCOL];
            auto issue_taps = [&](int cq, uint32_t *dst) {
                const int c8 = ES::CPW * h + 8 * cq;
                if (GC <= 8) {
                    const uint32_t col = (uint32_t)((c8 / GC) * W);
#pragma unroll
                    for (int m2 = 0; m2 < TP::NCOL / TP::PIECE; ++m2)
                        tmem_ld<TP::PIECE>(tl + col + m2 * TP::PIECE, dst + m2 * TP::PIECE);
                } else {
                    const uint32_t col = (uint32_t)((c8 / p.G) * W);
#pragma unroll
                    for (int k = 0; k < W; ++k) tmem_ld<1>(tl + col + k, dst + k);
                }
            };
            issue_taps(0, wr[0]);
#pragma unroll
            for (int cq = 0; cq < ES::CHUNKS; ++cq) {
                uint4 xu[W];
#pragma unroll
                for (int k = 0; k < W; ++k) xu[k] = lds128(xs + (xrow[k] ^ ((uint32_t)cq << 4)));
                float2 csv[4];
                const bool rot = rot_row && c_warp + 8 * cq < p.n_rot;
                if (ROPE) {
#pragma unroll
                    for (int m2 = 0; m2 < 4; ++m2) csv[m2] = csn[m2];
                    if (cq + 1 < ES::CHUNKS) load_cs(cq + 1);
                }
                tmem_wait_ld_regs(wr[cq & 1]);
                if (cq + 1 < ES::CHUNKS) issue_taps(cq + 1, wr[(cq + 1) & 1]);   // overlaps the math below
                float out[8];
                conv_chunk<W, GC>(wr[cq & 1], xu, out);
                if (rot) {
#pragma unroll
                    for (int m2 = 0; m2 < 4; ++m2) {
                        const float a = out[2 * m2], e = out[2 * m2 + 1];
                        out[2 * m2] = fmaf(a, csv[m2].x, -e * csv[m2].y);
                        out[2 * m2 + 1] = fmaf(a, csv[m2].y, e * csv[m2].x);
                    }
                }
                uint4 o;
                o.x = pack_bf16x2(out[0], out[1]);
                o.y = pack_bf16x2(out[2], out[3]);
                o.z = pack_bf16x2(out[4], out[5]);
                o.w = pack_bf16x2(out[6], out[7]);
                sts128(yw ^ ((uint32_t)cq << 4), o);
            }
            tc_fence_before();
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(bar.acce(a));
                mbar_arrive(bar.empty(s));
                tma_store_3d(&tm_y, ystage + yb * ES::YBUF, slice * kDt + ES::CPW * h, t0 + 32 * q, b);
                bulk_commit();
            }
            ++yc;
            slice += dslice;
            tt += dtl;
            if (slice >= p.n_slices) {
                slice -= p.n_slices;
                ++tt;
            }
            if (tt >= p.tiles_per_seq) {
                b += tt / p.tiles_per_seq;
                tt -= (tt / p.tiles_per_seq) * p.tiles_per_seq;
            }
            if ((s += ES::SETS) >= S) { s -= S; ++n; }
            if ((a += ES::SETS) >= p.nbuf) {
                m += a / p.nbuf;
                a -= (a / p.nbuf) * p.nbuf;
            }
        }
        if (lane == 0) bulk_wait_all();
        __syncwarp();
    }

    __syncthreads();
    if (warp == 1) {
        if (lane == 0) mbar_drain(bar.done(), 0, p.wt.wait_ns);
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, p.tmem_cols);
    }
}

template <int W, int GC, bool ROPE>
__global__ void __launch_bounds__(EpiShape<W, GC>::THREADS, 1)
k_tc_lowrank_fwd(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_z,
                 const __grid_constant__ CUtensorMap tm_u, const __grid_constant__ CUtensorMap tm_y,
                 const FwdParams p) {
    fwd_tiles<W, GC, ROPE, false>(tm_x, tm_z, tm_u, tm_y, nullptr, p);
}

template <int W, int GC>
__global__ void __launch_bounds__(EpiShape<W, GC, true>::THREADS, 1)
k_tc_decode_lowrank(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_z,
                    const __grid_constant__ CUtensorMap tm_u, const __grid_constant__ CUtensorMap tm_y,
                    const __grid_constant__ DecMaps dm, const FwdParams p) {
    fwd_tiles<W, GC, false, true>(tm_x, tm_z, tm_u, tm_y, &dm, p);
}

// ------------------------------------------------------------------ host side
namespace {

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
    std::call_once(g_encode_once, [] {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = (PFN_cuTensorMapEncodeTiled_v12000)fn;
    });
    return g_encode;
}

// Row-major bf16 tensor map; dims[0] is the contiguous dimension.
bool make_map(CUtensorMap *m, const void *ptr, int rank, const uint64_t *dims, const uint32_t *box,
              CUtensorMapSwizzle sw, CUtensorMapL2promotion promo = CU_TENSOR_MAP_L2_PROMOTION_L2_128B) {
    auto enc = encoder();
    if (!enc) return false;
    cuuint64_t gdim[3], gstride[2];
    cuuint32_t bdim[3], estr[3] = {1, 1, 1};
    uint64_t stride = 2;
    for (int i = 0; i < rank; ++i) {
        gdim[i] = dims[i];
        bdim[i] = box[i];
        if (i > 0) gstride[i - 1] = stride;
        stride *= dims[i];
    }
    const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void *>(ptr), gdim, gstride,
                           bdim, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, promo,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

int num_sms() {
    static int n[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return 148;
    if (!n[dev]) cudaDeviceGetAttribute(&n[dev], cudaDevAttrMultiProcessorCount, dev);
    return n[dev] > 0 ? n[dev] : 148;
}

bool is_pow2(int v) { return v > 0 && (v & (v - 1)) == 0; }

constexpr uint32_t kSmemLimit = 227 * 1024;

// dec: the decode step's layout (T = the number of sequences, B = 1; an x stage holds
// x_t and the W-1 window rows of 128 sequences).
bool plan_fwd(int B, int T, int D, int G, int W, int R, FwdParams &p, bool dec = false) {
    if (!(R == 16 || R == 32 || R == 64)) return false;
    if (D % kDt || !is_pow2(G) || G > 64 || W < 1 || W > 8) return false;
    p.B = B; p.T = T; p.D = D; p.G = G; p.R = R;
    p.slice_cols = (kDt / G) * W;
    if (p.slice_cols % 8) return false;           // U slice start must be 16-byte aligned for TMA
    p.n_pad = (p.slice_cols + 15) / 16 * 16;
    p.u_boxes = (p.n_pad + 63) / 64;
    p.tiles_per_seq = (T + kTt - 1) / kTt;
    p.n_slices = D / kDt;
    const long long nt = (long long)p.n_slices * B * p.tiles_per_seq;
    if (nt >= (1ll << 31)) return false;
    p.n_tiles = (int)nt;
    p.bufcols = p.n_pad;
    p.nbuf = (2 * p.n_pad <= 512) ? 2 : 1;
    int cols = 32;
    while (cols < p.nbuf * p.bufcols) cols *= 2;
    p.tmem_cols = cols;
    p.x_stage_tx = dec ? (uint32_t)W * kDecRow : (uint32_t)(kDt * 2 * (kTt + W - 1));
    p.x_stage_bytes = (p.x_stage_tx + 1023) / 1024 * 1024;
    p.z_stage_bytes = (uint32_t)(kTt * R * 2);
    p.u_bytes = (uint32_t)(p.u_boxes * R * 128);
    p.z_layout = R == 16 ? kSw32 : (R == 32 ? kSw64 : kSw128);
    const int ncol = G <= 8 ? (8 / G) * W : W;      // must match EpiShape / Taps
    p.nwg = (!dec && ncol <= 32 && DSC_FWD_SETS >= 2) ? 2 : 1;   // epilogue warp sets
    if (p.nbuf < p.nwg) p.nwg = p.nbuf;
    p.y_buf_bytes = (uint32_t)(32 * 32 * 2);
    p.off_z = 0;
    p.off_u = p.z_stage_bytes;
    p.op_bytes = (p.off_u + p.u_bytes + 1023) / 1024 * 1024;
    p.op_stages = kOpStages;
    p.off_op = 0;
    p.off_x = p.op_stages * p.op_bytes;
    // as deep an x ring as fits next to the operand ring and the y staging
    // (at least one stage per epilogue set; the decode step's single set can do with one)
    for (int st = kMaxXStages; st >= std::max(p.nwg, dec ? 1 : 2); --st) {
        const uint32_t off_y = p.off_x + st * p.x_stage_bytes;
        const uint32_t off_bar = off_y + 8 * p.nwg * 2 * p.y_buf_bytes;
        const uint32_t total = off_bar + kBarBytes + 16 + 1024;
        if (total <= kSmemLimit) {
            p.stages = st;
            p.off_y = off_y;
            p.off_bar = off_bar;
            return true;
        }
    }
    return false;
}

uint32_t smem_bytes(const FwdParams &p) { return p.off_bar + kBarBytes + 16 + 1024; }

// bf16 tensor map with explicit byte strides of dims 1.. (dims[0] contiguous).
bool make_map_strided(CUtensorMap *m, const void *ptr, const uint64_t (&dims)[3], const uint64_t (&strides)[2],
                      const uint32_t (&box)[3], CUtensorMapSwizzle sw) {
    auto enc = encoder();
    if (!enc) return false;
    cuuint64_t gdim[3] = {dims[0], dims[1], dims[2]}, gstride[2] = {strides[0], strides[1]};
    cuuint32_t bdim[3] = {box[0], box[1], box[2]}, estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), gdim, gstride, bdim, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int W, int GC>
cudaError_t launch_fwd_t(const CUtensorMap &mx, const CUtensorMap &mz, const CUtensorMap &mu,
                         const CUtensorMap &my, const FwdParams &p, cudaStream_t s) {
    auto kern = p.n_rot > 0 ? k_tc_lowrank_fwd<W, GC, true> : k_tc_lowrank_fwd<W, GC, false>;
    using ES = EpiShape<W, GC>;
    if (p.nwg != ES::SETS || p.y_buf_bytes != (uint32_t)ES::YBUF) return cudaErrorInvalidConfiguration;
    const uint32_t smem = smem_bytes(p);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int grid = std::min(p.n_tiles, num_sms());
    kern<<<grid, ES::THREADS, smem, s>>>(mx, mz, mu, my, p);
    return cudaGetLastError();
}

template <int W, int GC>
cudaError_t launch_dec_t(const CUtensorMap &mx, const CUtensorMap &mz, const CUtensorMap &mu,
                         const CUtensorMap &my, const DecMaps &dm, const FwdParams &p, cudaStream_t s) {
    auto kern = k_tc_decode_lowrank<W, GC>;
    using ES = EpiShape<W, GC, true>;
    if (p.nwg != ES::SETS || p.y_buf_bytes != (uint32_t)ES::YBUF) return cudaErrorInvalidConfiguration;
    const uint32_t smem = smem_bytes(p);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int grid = std::min(p.n_tiles, num_sms());
    kern<<<grid, ES::THREADS, smem, s>>>(mx, mz, mu, my, dm, p);
    return cudaGetLastError();
}

template <int W>
cudaError_t launch_dec_w(int G, const CUtensorMap &mx, const CUtensorMap &mz, const CUtensorMap &mu,
                         const CUtensorMap &my, const DecMaps &dm, const FwdParams &p, cudaStream_t s) {
    switch (G) {
        case 1: return launch_dec_t<W, 1>(mx, mz, mu, my, dm, p, s);
        case 2: return launch_dec_t<W, 2>(mx, mz, mu, my, dm, p, s);
        case 4: return launch_dec_t<W, 4>(mx, mz, mu, my, dm, p, s);
        case 8: return launch_dec_t<W, 8>(mx, mz, mu, my, dm, p, s);
        default: return launch_dec_t<W, 16>(mx, mz, mu, my, dm, p, s);
    }
}

template <int W>
cudaError_t launch_fwd_w(int G, const CUtensorMap &mx, const CUtensorMap &mz, const CUtensorMap &mu,
                         const CUtensorMap &my, const FwdParams &p, cudaStream_t s) {
    switch (G) {
        case 1: return launch_fwd_t<W, 1>(mx, mz, mu, my, p, s);
        case 2: return launch_fwd_t<W, 2>(mx, mz, mu, my, p, s);
        case 4: return launch_fwd_t<W, 4>(mx, mz, mu, my, p, s);
        case 8: return launch_fwd_t<W, 8>(mx, mz, mu, my, p, s);
        default: return launch_fwd_t<W, 16>(mx, mz, mu, my, p, s);
    }
}

}  // namespace
}  // namespace tc

bool tc_lowrank_fwd_supported(int B, int T, int D, int G, int W, int R, bool bf16) {
    tc::FwdParams p;
    return bf16 && tc::plan_fwd(B, T, D, G, W, R, p);
}

cudaError_t launch_tc_lowrank_fwd(const void *x, const void *z, const void *U, void *y, int B, int T,
                                  int D, int G, int W, int R, cudaStream_t s, const float *cs, int dh, int n_rot) {
    using namespace tc;
    FwdParams p;
    if (!plan_fwd(B, T, D, G, W, R, p)) return cudaErrorNotSupported;
    p.cs = cs;
    p.dh = dh;
    p.n_rot = cs ? n_rot : 0;
    take_wait_test(&p.wt.wait_ns, &p.wt.withhold_cta);
    CUtensorMap mx, mz, mu, my;
    const uint64_t dx[3] = {(uint64_t)D, (uint64_t)T, (uint64_t)B};
    const uint32_t bx[3] = {(uint32_t)kDt, (uint32_t)(kTt + W - 1), 1};
    const uint64_t dz[3] = {(uint64_t)R, (uint64_t)T, (uint64_t)B};
    const uint32_t bz[3] = {(uint32_t)R, (uint32_t)kTt, 1};
    const uint64_t du[2] = {(uint64_t)(D / G) * W, (uint64_t)R};
    const uint32_t bu[2] = {64, (uint32_t)R};
    const uint32_t by[3] = {32, 32, 1};
    const CUtensorMapSwizzle zsw = R == 16 ? CU_TENSOR_MAP_SWIZZLE_32B
                                           : (R == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B);
    const CUtensorMapL2promotion xpromo =
        DSC_X_L2_PROMO == 256 ? CU_TENSOR_MAP_L2_PROMOTION_L2_256B : CU_TENSOR_MAP_L2_PROMOTION_L2_128B;
    if (!make_map(&mx, x, 3, dx, bx, CU_TENSOR_MAP_SWIZZLE_128B, xpromo) ||
        !make_map(&mz, z, 3, dz, bz, zsw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B) ||
        !make_map(&mu, U, 2, du, bu, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B) ||
        !make_map(&my, y, 3, dx, by, CU_TENSOR_MAP_SWIZZLE_64B)) {
        set_last_error("dsc_fwd_lowrank: cuTensorMapEncodeTiled failed");
        return cudaErrorInvalidValue;
    }
    switch (W) {
        case 1: return launch_fwd_w<1>(G, mx, mz, mu, my, p, s);
        case 2: return launch_fwd_w<2>(G, mx, mz, mu, my, p, s);
        case 3: return launch_fwd_w<3>(G, mx, mz, mu, my, p, s);
        case 4: return launch_fwd_w<4>(G, mx, mz, mu, my, p, s);
        case 5: return launch_fwd_w<5>(G, mx, mz, mu, my, p, s);
        case 6: return launch_fwd_w<6>(G, mx, mz, mu, my, p, s);
        case 7: return launch_fwd_w<7>(G, mx, mz, mu, my, p, s);
        default: return launch_fwd_w<8>(G, mx, mz, mu, my, p, s);
    }
}

bool tc_decode_lowrank_supported(int B, int D, int G, int W, int R, bool bf16) {
    tc::FwdParams p;
    return bf16 && B > 0 && tc::plan_fwd(1, B, D, G, W, R, p, true);
}

cudaError_t launch_tc_decode_lowrank(const void *x, const void *z, const void *U, void *st, void *y, int B, int D,
                                     int G, int W, int R, cudaStream_t s) {
    using namespace tc;
    FwdParams p;
    if (!plan_fwd(1, B, D, G, W, R, p, true)) return cudaErrorNotSupported;
    p.cs = nullptr;
    p.dh = 0;
    p.n_rot = 0;
    take_wait_test(&p.wt.wait_ns, &p.wt.withhold_cta);
    CUtensorMap mx, mz, mu, my;
    DecMaps dm;
    memset(&dm, 0, sizeof(dm));
    const uint64_t dx[3] = {(uint64_t)D, (uint64_t)B, 1};
    const uint32_t bx[3] = {(uint32_t)kDt, (uint32_t)kTt, 1};
    const uint64_t dz[3] = {(uint64_t)R, (uint64_t)B, 1};
    const uint32_t bz[3] = {(uint32_t)R, (uint32_t)kTt, 1};
    const uint64_t du[2] = {(uint64_t)(D / G) * W, (uint64_t)R};
    const uint32_t bu[2] = {64, (uint32_t)R};
    const uint32_t by[3] = {32, 32, 1};
    const CUtensorMapSwizzle zsw = R == 16 ? CU_TENSOR_MAP_SWIZZLE_32B
                                           : (R == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B);
    bool ok = make_map(&mx, x, 3, dx, bx, CU_TENSOR_MAP_SWIZZLE_128B) &&
              make_map(&mz, z, 3, dz, bz, zsw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B) &&
              make_map(&mu, U, 2, du, bu, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B) &&
              make_map(&my, y, 3, dx, by, CU_TENSOR_MAP_SWIZZLE_64B);
    if (ok && W > 1) {
        // the window [B, W-1, D] as dims {D, B, W-1}: sequence stride (W-1)*D, row stride D
        const uint64_t ds[3] = {(uint64_t)D, (uint64_t)B, (uint64_t)(W - 1)};
        const uint64_t ss[2] = {(uint64_t)(W - 1) * D * 2, (uint64_t)D * 2};
        const uint32_t bl[3] = {(uint32_t)kDt, (uint32_t)kTt, (uint32_t)(W - 1)};
        const uint32_t bs[3] = {(uint32_t)kDt, (uint32_t)kTt, (uint32_t)(W > 2 ? W - 2 : 1)};
        const uint32_t bp[3] = {(uint32_t)kDt, (uint32_t)kTt, 1};
        ok = make_map_strided(&dm.load, st, ds, ss, bl, CU_TENSOR_MAP_SWIZZLE_128B) &&
             (W == 2 || make_map_strided(&dm.shift, st, ds, ss, bs, CU_TENSOR_MAP_SWIZZLE_128B)) &&
             make_map_strided(&dm.push, st, ds, ss, bp, CU_TENSOR_MAP_SWIZZLE_128B);
    }
    if (!ok) {
        set_last_error("dsc_decode_step_lowrank: cuTensorMapEncodeTiled failed");
        return cudaErrorInvalidValue;
    }
    switch (W) {
        case 1: return launch_dec_w<1>(G, mx, mz, mu, my, dm, p, s);
        case 2: return launch_dec_w<2>(G, mx, mz, mu, my, dm, p, s);
        case 3: return launch_dec_w<3>(G, mx, mz, mu, my, dm, p, s);
        case 4: return launch_dec_w<4>(G, mx, mz, mu, my, dm, p, s);
        case 5: return launch_dec_w<5>(G, mx, mz, mu, my, dm, p, s);
        case 6: return launch_dec_w<6>(G, mx, mz, mu, my, dm, p, s);
        case 7: return launch_dec_w<7>(G, mx, mz, mu, my, dm, p, s);
        default: return launch_dec_w<8>(G, mx, mz, mu, my, dm, p, s);
    }
}

unsigned read_device_fault(bool reset) {
    unsigned v = 0;
    if (cudaMemcpyFromSymbol(&v, tc::g_fault, sizeof(v)) != cudaSuccess) return 0xffffffffu;
    if (reset) {
        const unsigned z = 0;
        cudaMemcpyToSymbol(tc::g_fault, &z, sizeof(z));
    }
    return v | (read_device_fault_bwd(reset) << 16);
}

}  // namespace dsc
