// Tensor-core (tcgen05 / TMEM / TMA) backward of the fused low-rank causal dynamic
// short convolution on sm_100a.
//
// Chain rule through "Convolucoes Curtas Dinamicas Melhoram Transformers" (Metodologia:
// Mecanismo y_t = x_t + sum_k w(t)_k x_{t-k}; Parametrizacao 1: w(t) = z_t U):
//   dx[t,c]   = dy[t,c] + sum_k w[t+k, g(c), k] dy[t+k, c]
//   dw[t,g,k] = sum_{c in g} dy[t,c] x[t-k,c]               (on chip only)
//   dz[t,r]   = sum_j dw[t,j] U[r,j]
//   dU[r,j]   = sum_t z[t,r] dw[t,j]
// The filters are recomputed from z and U rather than stored (storing them would move
// W/G times the bytes of x), and dw never leaves the chip ("Implementacao de
// Treinamento Eficiente": the kernels write only the final results to HBM).
//
// Work tile = 128 tokens of one sequence ("token tile") x one 64-channel slice.
//
// Schedule (one persistent CTA per SM, cooperative launch).  The grid is A x Bg
// CTAs: CTA (a, b) owns the token tiles of range a and the S slices of group b, and
// walks them token tile by token tile, its S slices innermost.  Hence
//   - dz of a token tile accumulates over the CTA's S slices in TMEM and leaves the
//     CTA once, added into dz with fp32 vector reductions in L2 (the Bg slice groups'
//     additions land in whatever order they arrive: dz is reproducible to rounding,
//     not bitwise);
//   - dU of each of its slices accumulates over all its token tiles in TMEM and
//     leaves the CTA once, as one partial of A; after the last tile the A partials of
//     each slice group are summed in a fixed order (a counter per group says when all
//     are written), so dU and dx are bitwise deterministic.
//
// Per tile (token tile m, slice s) the CTA's warps do:
//   warp 0      TMA: dy and x tiles (3-stage ring), z once per token tile, the
//               tap-major U slice Up (resident when the CTA has at most two slices);
//               TMA store of dx from the stage once the epilogue has written it there
//   warp 1      recompute: one MMA per tap k with the z tile shifted by k rows,
//                 Wk[t, g] = sum_r z[t0+t+k, r] Up[r, k*NG+g],
//               so TMEM lane t holds w[t+k, g, k] for every k
//   warp 2      dz[m] += dw Up^T  (A = dw tile, B = Up slice; M=128 tokens, N=R) and
//               dU^T[s] += dw^T z  (A = dw tile read MN-major, B = z; M=128 columns)
//   warp 3      idle (keeps the epilogue warps four to a sub-partition)
//   warps 4-19  epilogue, one token row per thread, 16 channels per warp:
//                 A2: dw (bf16) into the shared-memory dw tile;
//                 A1: dx, written over the stage's x tile (dead after A2);
//                 after a token tile's last slice: its dz sum, added into dz
// The recompute of tile i runs during A2 of tile i, and the dz/dU MMAs of tile i
// during A1 of tile i.  Every wait is bounded (one second); a wait that runs out
// makes the CTA leave its loops, record a fault code and free its TMEM.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstdio>
#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"

namespace dsc {
namespace tcb {

using namespace dsc::tc;

__device__ unsigned int g_fault_bwd = 0;

constexpr int kTt = 128;
constexpr int kDt = 64;
constexpr int kEpiWarps = 16;                   // 4 TMEM lane quarters x 4 channel groups
constexpr int kCPW = kDt / 4;                   // channels per epilogue warp
// Warp roles.  Warps 0-3 sit on the SM's four sub-partitions, one each, and the
// epilogue warps 4-19 four to a sub-partition; 20 warps keep 96 registers a thread.
constexpr int kRecWarp = 1;
constexpr int kMmaWarp = 2;                     // dz and dU MMAs (warp 3 idles)
constexpr int kEpi0 = 4;
constexpr int kThreads = 32 * (kEpi0 + kEpiWarps);
constexpr int kMaxStages = 3;

struct BwdParams {
    int B, T, D, G, W, R;
    int NGs;                  // filter groups per slice (64/G)
    int NGp;                  // columns per tap block in Up, the dw tile and TMEM (Cols::NB)
    int SC;                   // filter columns of U per slice (NGs*W)
    int SCq;                  // columns per slice in the tap-major layout (Cols::SCQ)
    int SCp;                  // SCq rounded up to 128 (dU^T M-blocks)
    int n_slices, tiles_per_seq, n_tt;
    int A, Bg;                // token ranges x slice groups = grid
    int u_boxes;              // TMA boxes of 64 Up columns per slice
    int stages, nU;           // ring depth; Up buffers (1 or 2)
    uint32_t rows;            // tile rows incl. halo: 128 + W - 1
    uint32_t xy_tile_bytes;   // one dy or x tile (rows x 128 B), 1024-aligned
    uint32_t z_slab;          // stride of the 8-wide z slabs (rows x 16 B, rounded up to 128)
    uint32_t z_bytes;         // one z buffer (R/8 slabs), 1024-aligned
    uint32_t u_bytes;         // one Up buffer
    uint32_t stage_bytes;     // dy tile + x tile
    uint32_t off_z, off_u, off_dw, off_bar;
    uint32_t tm_w, tm_dz, tm_du, tmem_cols;   // TMEM column map
    float *du_part;           // [A][R][N]
    unsigned *flag_du;        // [Bg]   dU partials written per slice group (16 per CTA)
    const float *cs;          // RoPE table [T][dh/2][2] (cos, sin): dy arrives rotated, or null
    int dh, n_rot;            // RoPE head size; channels [0, n_rot) rotated (0: none)
    float *dz;                // [B*T][R]
    float *dU;                // [R][N]
    WaitTest wt;
};

struct Bars {
    uint32_t base;
    __device__ uint32_t full(int s) const { return base + 8 * s; }
    __device__ uint32_t dxr(int s) const { return base + 8 * (3 + s); }
    __device__ uint32_t zfull(int z) const { return base + 8 * (6 + z); }
    __device__ uint32_t zempty(int z) const { return base + 8 * (8 + z); }
    __device__ uint32_t ufull(int u) const { return base + 8 * (10 + u); }
    __device__ uint32_t uempty(int u) const { return base + 8 * (12 + u); }
    __device__ uint32_t wfull() const { return base + 8 * 14; }
    __device__ uint32_t wempty() const { return base + 8 * 15; }
    __device__ uint32_t dwready() const { return base + 8 * 16; }
    __device__ uint32_t dwfree() const { return base + 8 * 17; }
    __device__ uint32_t dzfull(int d) const { return base + 8 * (18 + d); }
    __device__ uint32_t dzempty(int d) const { return base + 8 * (20 + d); }
    __device__ uint32_t dufull() const { return base + 8 * 22; }
    __device__ uint32_t done() const { return base + 8 * 23; }
    __device__ uint32_t xdead() const { return base + 8 * 24; }
    __device__ uint32_t dyrot() const { return base + 8 * 25; }
};
constexpr uint32_t kBarBytes = 8 * 26;

__device__ __forceinline__ void unpack8(const uint4 &u, float (&v)[8]) {
    v[0] = bf16_lo(u.x); v[1] = bf16_hi(u.x);
    v[2] = bf16_lo(u.y); v[3] = bf16_hi(u.y);
    v[4] = bf16_lo(u.z); v[5] = bf16_hi(u.z);
    v[6] = bf16_lo(u.w); v[7] = bf16_hi(u.w);
}

// Column layout of the tap-major filter blocks (the Up copy of U, the dw tile and the
// recomputed filters in TMEM).  For G <= 4 a tap block has one column per filter group
// of the slice (64/G >= 16).  For G >= 8 the block is padded to 16 columns, the MMA's
// smallest N and a 32-byte descriptor step; and for G >= 32, where a group would span
// several epilogue warps, each warp's 16 channels form a "virtual group" with a copy of
// the group's U column: dz = dw Up^T sums the virtual groups by itself, and the dU
// columns of a group's virtual groups are added when dU is read out.
template <int W, int G>
struct Cols {
    static constexpr int GV = G < 16 ? G : 16;       // channels per (virtual) group
    static constexpr int NGV = 64 / GV;              // (virtual) groups per slice
    static constexpr int NB = NGV < 16 ? 16 : NGV;   // columns per tap block
    static constexpr int SCQ = NB * W;               // columns per slice
    static constexpr int NMB = (SCQ + 127) / 128;    // dU^T M-blocks per slice
    static constexpr int VPR = G / GV;               // virtual groups per real group
};

__device__ __forceinline__ void sts16(uint32_t addr, uint16_t v) {
    asm volatile("st.shared.u16 [%0], %1;" ::"r"(addr), "h"(v) : "memory");
}
__device__ __forceinline__ void sts32(uint32_t addr, uint32_t v) {
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ void sts64(uint32_t addr, uint32_t a, uint32_t b) {
    asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(addr), "r"(a), "r"(b) : "memory");
}

// ------------------------------------------------------------------ global counters
// A writer's stores become visible before its count: the writers synchronise with the
// publishing warp (an mbarrier), which fences at gpu scope and then adds (relaxed; the
// fence before it makes the pair a release).  A reader polls with acquire
// semantics (every lane), then reads the data through L2.
__device__ __forceinline__ void fence_gpu() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }

__device__ __forceinline__ void red_release_add(unsigned *p, unsigned v) {
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// dst[0..3] += v (fp32, one vector reduction in L2).
__device__ __forceinline__ void red_add_v4(float *dst, const uint32_t (&v)[4]) {
    asm volatile("red.relaxed.gpu.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dst), "f"(__uint_as_float(v[0])),
                 "f"(__uint_as_float(v[1])), "f"(__uint_as_float(v[2])), "f"(__uint_as_float(v[3]))
                 : "memory");
}

__device__ __forceinline__ unsigned ld_acquire(const unsigned *p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Waits until *p >= target.  Gives up like mbar_wait: after kWaitLimitNs, or as soon
// as another warp of the CTA has given up.
__device__ __forceinline__ bool wait_count(const unsigned *p, unsigned target, volatile int *abort,
                                           unsigned code, unsigned long long limit_ns) {
    if (ld_acquire(p) >= target) return true;
    const unsigned long long t0 = globaltimer();
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 16; ++i) {
            __nanosleep(100);
            if (ld_acquire(p) >= target) return true;
        }
        if (*abort) return false;
        if (globaltimer() - t0 > limit_ns) {
            *abort = 1;
            atomicOr(&g_fault_bwd, code);
            return false;
        }
    }
}

// Which token tiles and slices a CTA owns.
struct Span {
    int a, b;                 // token range, slice group
    int m0, m1, s0, s1;       // token tiles [m0, m1), slices [s0, s1)
    __device__ int S() const { return s1 - s0; }
    __device__ int tiles() const { return (m1 - m0) * (s1 - s0); }
};
// Position in a CTA's walk over its tiles (token tiles outermost, its S slices
// innermost), advanced by increments so that the loops divide by nothing.
struct Walk {
    int i = 0;                // tile
    int j = 0, mz = 0;        // slice within the segment, token tile within the CTA
    int st = 0, n = 0;        // ring stage and round
    int b, tt;                // sequence and tile within it of token tile m0 + mz
    __device__ Walk(int m0, int tiles_per_seq) {
        b = m0 / tiles_per_seq;
        tt = m0 - b * tiles_per_seq;
    }
    __device__ int t0() const { return tt * kTt; }
    __device__ void next(int S, int NST, int tiles_per_seq) {
        ++i;
        if (++st == NST) { st = 0; ++n; }
        if (++j == S) {
            j = 0;
            ++mz;
            if (++tt == tiles_per_seq) { tt = 0; ++b; }
        }
    }
};

__device__ __forceinline__ Span span_of(const BwdParams &p) {
    Span s;
    s.a = (int)blockIdx.x / p.Bg;
    s.b = (int)blockIdx.x - s.a * p.Bg;
    s.m0 = (int)((long long)s.a * p.n_tt / p.A);
    s.m1 = (int)((long long)(s.a + 1) * p.n_tt / p.A);
    s.s0 = (int)((long long)s.b * p.n_slices / p.Bg);
    s.s1 = (int)((long long)(s.b + 1) * p.n_slices / p.Bg);
    return s;
}

// ROPE: the instantiation that rotates dy back (dsc_bwd_lowrank_rope); the plain one has
// no RoPE code.
template <int W, int G, bool ROPE>
__global__ void __launch_bounds__(kThreads, 1)
k_tc_lowrank_bwd(const __grid_constant__ CUtensorMap tm_dy, const __grid_constant__ CUtensorMap tm_x,
                 const __grid_constant__ CUtensorMap tm_z, const __grid_constant__ CUtensorMap tm_u,
                 const __grid_constant__ CUtensorMap tm_dx, const BwdParams p) {
    using CL = Cols<W, G>;
    constexpr int GV = CL::GV;
    constexpr int NG8 = GV <= 8 ? 8 / GV : 1;   // (virtual) groups in one 8-channel chunk
    constexpr int NGS = kDt / G;                 // filter groups per slice
    constexpr int CH = kCPW / 8;        // 16-byte chunks of a warp's channels in a row
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const uint32_t sb = smem_u32(smem);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const Bars bar{sb + p.off_bar};
    uint32_t *tmem_holder = (uint32_t *)(smem + p.off_bar + kBarBytes);
    volatile int *abort = (volatile int *)(smem + p.off_bar + kBarBytes + 8);
    const Span sp = span_of(p);
    const int S = sp.S();
    const int nt = sp.tiles();
    const int NST = p.stages;
    const bool u_res = S <= p.nU;       // Up slices stay resident: buffer j holds slice s0+j

    if (threadIdx.x == 0) {
        for (int s = 0; s < NST; ++s) {
            mbar_init(bar.full(s), 1);
            mbar_init(bar.dxr(s), kEpiWarps);
        }
        for (int z = 0; z < 2; ++z) {
            mbar_init(bar.zfull(z), 1);
            mbar_init(bar.zempty(z), 2);        // recompute and dz/dU streams
            mbar_init(bar.ufull(z), 1);
            mbar_init(bar.uempty(z), 2);        // recompute and dz/dU streams
            mbar_init(bar.dzfull(z), 1);
            mbar_init(bar.dzempty(z), kEpiWarps);
        }
        mbar_init(bar.wfull(), 1);
        mbar_init(bar.wempty(), kEpiWarps);
        mbar_init(bar.dwready(), kEpiWarps);
        mbar_init(bar.dwfree(), 1);
        mbar_init(bar.dufull(), 1);
        mbar_init(bar.done(), 2);               // recompute and dz/dU streams
        mbar_init(bar.xdead(), kEpiWarps);      // every epilogue warp is past A2
        mbar_init(bar.dyrot(), kEpiWarps);      // every epilogue warp has un-rotated its dy rows
        *abort = 0;
        fence_barrier_init();
    }
    // Columns of the dw tile that no epilogue warp writes (the padding of the last
    // 128-column M-block, and the padding of each tap block when G >= 8) must read as zero.
    if (G >= 8 || p.SCp > p.SCq) {
        for (uint32_t o = threadIdx.x * 16; o < (uint32_t)(p.SCp / 64) * 16384u; o += kThreads * 16) {
            const uint32_t atom = o / 16384u;
            if (G >= 8 || (int)(atom * 64) + 64 > p.SCq) sts128(sb + p.off_dw + o, make_uint4(0, 0, 0, 0));
        }
        fence_proxy_async_smem();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch(&tm_dy);
        tma_prefetch(&tm_x);
        tma_prefetch(&tm_z);
        tma_prefetch(&tm_u);
        tma_prefetch(&tm_dx);
    }
    if (warp == kRecWarp) {
        tmem_alloc(smem_u32(tmem_holder), p.tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    if (warp == 0) {
        // ---------------------------------------------------------- TMA producer
        if (lane == 0) {
            const uint32_t tx_xy = 2 * p.rows * 128;
            const uint32_t tx_z = (uint32_t)(p.R / 8) * p.rows * 16;
            auto load_up = [&](int ub, int slice) {
                mbar_arrive_expect_tx(bar.ufull(ub), p.u_bytes);
                const uint32_t ud = sb + p.off_u + ub * p.u_bytes;
                for (int bx = 0; bx < p.u_boxes; ++bx)
                    tma_load_2d(ud + bx * (uint32_t)(p.R * 128), &tm_u, bar.ufull(ub), slice * p.SCq + 64 * bx, 0);
            };
            auto store_dx = [&](int i) {      // dx of tile i, from its stage's x region
                const int m = sp.m0 + i / S, slice = sp.s0 + i % S;
                const int b = m / p.tiles_per_seq, t0 = (m - b * p.tiles_per_seq) * kTt;
                tma_store_3d(&tm_dx, sb + (i % NST) * p.stage_bytes + p.xy_tile_bytes, slice * kDt, t0, b);
                bulk_commit();
            };
            int issued = 0, zissued = 0, uissued = 0;
            bool ok = true;
            if (u_res)
                for (int j = 0; j < S; ++j) { load_up(j, sp.s0 + j); ++uissued; }
            for (Walk w(sp.m0, p.tiles_per_seq); w.i < nt && ok; w.next(S, NST, p.tiles_per_seq)) {
                const int i = w.i, st = w.st, n = w.n, j = w.j, mz = w.mz;
                const int slice = sp.s0 + j, b = w.b, t0 = w.t0();
                if (i >= NST) {
                    // the stage is free once tile i-NST's dx, written over its x tile, is stored
                    if (!mbar_wait(bar.dxr(st), (n - 1) & 1, abort, 1u, &g_fault_bwd, p.wt.wait_ns)) { ok = false; break; }
                    store_dx(i - NST);
                    bulk_wait_read<0>();
                }
                if (j == 0) {
                    const int zb = mz & 1;
                    if (!mbar_wait(bar.zempty(zb), ((mz >> 1) & 1) ^ 1, abort, 2u, &g_fault_bwd, p.wt.wait_ns)) { ok = false; break; }
                    mbar_arrive_expect_tx(bar.zfull(zb), tx_z);
                    const uint32_t zd = sb + p.off_z + zb * p.z_bytes;
                    for (int r8 = 0; r8 < p.R / 8; ++r8)
                        tma_load_3d(zd + r8 * p.z_slab, &tm_z, bar.zfull(zb), 8 * r8, t0, b);
                    ++zissued;
                }
                if (!u_res) {
                    const int ub = i & 1;
                    if (!mbar_wait(bar.uempty(ub), ((i >> 1) & 1) ^ 1, abort, 2u, &g_fault_bwd, p.wt.wait_ns)) { ok = false; break; }
                    load_up(ub, slice);
                    ++uissued;
                }
                ++issued;
                if (i == 0 && (int)blockIdx.x == p.wt.withhold_cta) continue;   // test hook: no loads
                mbar_arrive_expect_tx(bar.full(st), tx_xy);
                const uint32_t sd = sb + st * p.stage_bytes;
                tma_load_3d(sd, &tm_dy, bar.full(st), slice * kDt, t0, b);
                tma_load_3d(sd + p.xy_tile_bytes, &tm_x, bar.full(st), slice * kDt, t0 - (W - 1), b);
            }
            if (ok) {
                for (int i = (nt > NST ? nt - NST : 0); i < nt; ++i) {
                    if (!mbar_wait(bar.dxr(i % NST), (i / NST) & 1, abort, 1u, &g_fault_bwd, p.wt.wait_ns)) break;
                    store_dx(i);
                }
            }
            bulk_wait_all();
            // Let every load this warp issued land before the CTA can exit (matters only
            // when another warp gave up early; otherwise all of them were consumed).
            for (int i = (issued > NST ? issued - NST : 0); i < issued; ++i)
                mbar_drain(bar.full(i % NST), (i / NST) & 1, p.wt.wait_ns);
            for (int z = (zissued > 2 ? zissued - 2 : 0); z < zissued; ++z)
                mbar_drain(bar.zfull(z & 1), (z >> 1) & 1, p.wt.wait_ns);
            if (u_res) {
                for (int u = 0; u < uissued; ++u) mbar_drain(bar.ufull(u), 0, p.wt.wait_ns);
            } else {
                for (int u = (uissued > 2 ? uissued - 2 : 0); u < uissued; ++u)
                    mbar_drain(bar.ufull(u & 1), (u >> 1) & 1, p.wt.wait_ns);
            }
        }
        __syncwarp();
    } else if (warp == kRecWarp) {
        // ---------------------------------------------------------- MMA issuer: recompute
        // Each MMA warp waits warp-uniformly; one elected lane then issues a tile's
        // tcgen05 instructions in a row, descriptors advancing by adds to their start field.
        // Tile i's filters are recomputed once the epilogue has read those of tile i-1:
        //   Wk[t, g] = sum_r z[t0+t+k, r] Up[r, k*NB+g], one MMA chain per tap with the z
        //   tile shifted by k rows (A: z, K-major; B: Up, MN-major).
        const uint64_t t_zk = desc_tmpl(p.z_slab, 128, kSwNone);               // z, K-major, no swizzle
        const uint64_t t_u_mn = desc_tmpl((uint32_t)(p.R * 128), 1024, kSw128);  // Up as MN-major B
        const uint32_t i_rec = idesc_bf16(128, CL::NB, false, true);
        const int ksr = p.R / 16;
        const uint32_t ubox = (uint32_t)(p.R * 128);
        const uint64_t st_zk = (2 * p.z_slab) >> 4;   // 16 more z columns (start field units)
        for (Walk w(sp.m0, p.tiles_per_seq); w.i < nt; w.next(S, NST, p.tiles_per_seq)) {
            const int i = w.i, j = w.j, mz = w.mz, zb = mz & 1;
            const int ub = u_res ? j : (i & 1);
            const int upar = u_res ? 0 : ((i >> 1) & 1);
            if (j == 0 && !warp_wait(bar.zfull(zb), (mz >> 1) & 1, abort, 4u, &g_fault_bwd, p.wt.wait_ns)) break;
            if (!warp_wait(bar.ufull(ub), upar, abort, 4u, &g_fault_bwd, p.wt.wait_ns)) break;
            if (!warp_wait(bar.wempty(), (i & 1) ^ 1, abort, 16u, &g_fault_bwd, p.wt.wait_ns)) break;
            tc_fence_after();
            const uint32_t zs = sb + p.off_z + zb * p.z_bytes;
            const uint32_t us = sb + p.off_u + ub * p.u_bytes;
            if (elect_one()) {      // one lane issues the tile's MMAs and commits
#pragma unroll
                for (int k = 0; k < W; ++k) {
                    const int col0 = k * CL::NB;
                    uint64_t da = desc_at(t_zk, zs + 16 * k);
                    uint64_t db = desc_at(t_u_mn, us + (col0 / 64) * ubox + (col0 % 64) * 2);
                    const uint32_t d = tmem + p.tm_w + k * CL::NB;
                    for (int kk = 0; kk < ksr; ++kk) {
                        mma_bf16_ss(d, da, db, i_rec, kk > 0 ? 1u : 0u);
                        da += st_zk;
                        db += 2048u >> 4;
                    }
                }
                mma_commit(bar.wfull());
                if (j == S - 1) mma_commit(bar.zempty(zb));
                if (!u_res) mma_commit(bar.uempty(ub));
            }
            __syncwarp();
        }
        if (elect_one()) mma_commit(bar.done());
        __syncwarp();
    } else if (warp >= kEpi0) {
        // ---------------------------------------------------------- epilogue
        const int ew = warp - kEpi0;
        const int q = warp & 3;              // TMEM lane quarter == token rows 32q..32q+31
        const int h = ew >> 2;               // channel group of the slice (kCPW channels)
        const int row = 32 * q + lane;
        // dy rows r = row + k and x rows r = row + W-1-k of the 128-byte-swizzled tiles;
        // dx of row `row` is written to row `row` of the x tile
        uint32_t dyr[W], xr[W];
#pragma unroll
        for (int k = 0; k < W; ++k) {
            uint32_t r = (uint32_t)(row + k);
            dyr[k] = (r * 128u) ^ ((r & 7u) << 4) ^ ((uint32_t)(CH * h) << 4);
            r = (uint32_t)(row + (W - 1) - k);
            xr[k] = (r * 128u) ^ ((r & 7u) << 4) ^ ((uint32_t)(CH * h) << 4);
        }
        const uint32_t dxr0 = ((uint32_t)row * 128u) ^ (((uint32_t)row & 7u) << 4) ^ ((uint32_t)(CH * h) << 4);
        // dw^T shared-memory tile: MN-major, 128B swizzle, atoms of 64 columns x 128 rows
        const uint32_t dwrow = sb + p.off_dw + (uint32_t)row * 128u;
        const uint32_t dwsw = (uint32_t)(row & 7) << 4;
        const uint32_t tl = tmem + ((uint32_t)(32 * q) << 16);
        const int nc = p.R / 4;              // dz columns a warp reads out (its group's share)

        // dz of token tile mz summed over this CTA's slices, added into dz (fp32 vector
        // reductions in L2; dz starts at zero, written by the U reorder kernel).
        auto dz_out = [&](int mz, int b, int t0) -> bool {
            const int db = mz & 1;
            if (!warp_wait(bar.dzfull(db), (mz >> 1) & 1, abort, 256u, &g_fault_bwd, p.wt.wait_ns)) return false;
            tc_fence_after();
            const int tok = t0 + row;
            float *dst = p.dz + ((size_t)b * p.T + tok) * p.R + h * nc;
            const uint32_t src = tl + p.tm_dz + db * p.R + h * nc;
#pragma unroll 1
            for (int c0 = 0; c0 < nc; c0 += 8) {
                uint32_t v[8];
                if (nc >= 8) {
                    tmem_ld<8>(src + c0, v);
                } else {
                    tmem_ld<4>(src + c0, v);
                    v[4] = v[5] = v[6] = v[7] = 0u;
                }
                tmem_wait_ld_regs(v);
                if (nc == 8) {
                    // a lane holds 32 contiguous bytes of its row; regrouped so that each
                    // reduction covers 16 rows x 32 bytes (16 sectors) instead of 32 rows
                    // x 16 bytes (32 sectors): lane l adds half l&1 of row 16*ps + l/2
#pragma unroll
                    for (int ps = 0; ps < 2; ++ps) {
                        const int sl = 16 * ps + (lane >> 1), hf = lane & 1;
                        uint32_t u[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const uint32_t lo = __shfl_sync(0xffffffffu, v[e], sl);
                            const uint32_t hi = __shfl_sync(0xffffffffu, v[4 + e], sl);
                            u[e] = hf ? hi : lo;
                        }
                        const int rt = t0 + 32 * q + sl;
                        if (rt < p.T) red_add_v4(p.dz + ((size_t)b * p.T + rt) * p.R + h * nc + c0 + 4 * hf, u);
                    }
                } else if (tok < p.T) {
                    red_add_v4(dst + c0, *reinterpret_cast<const uint32_t(*)[4]>(v));
                    if (nc >= 8) red_add_v4(dst + c0 + 4, *reinterpret_cast<const uint32_t(*)[4]>(v + 4));
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar.dzempty(db));
            return true;
        };

        bool ok = true;
        int pb = 0, pt0 = 0;                 // sequence and first token of the previous token tile
        int nrot = 0;                        // dyrot phases waited for
        for (Walk w(sp.m0, p.tiles_per_seq); w.i < nt; w.next(S, NST, p.tiles_per_seq)) {
            const int i = w.i, j = w.j, mz = w.mz;
            const int st = w.st, n = w.n;
            if (!warp_wait(bar.full(st), n & 1, abort, 64u, &g_fault_bwd, p.wt.wait_ns)) { ok = false; break; }
            const uint32_t dys = sb + st * p.stage_bytes, xs = dys + p.xy_tile_bytes;

            // ---- RoPE (when on): dy arrives as the gradient of the rotated output and is
            // rotated back in the stage's dy tile (the transpose: pair (2i, 2i+1) by minus
            // its angle) before A1, which reads neighbours' rows, waits for every warp
            // (dyrot).  For G >= 8 each thread rotates its own row here (lanes 0..W-2 of
            // quarter 0 also the tile's W-1 future-halo rows) and A2 reads only that row;
            // for G < 8 A2's threads rotate the rows they read (below).
            constexpr bool kRowPairs = G < 8;
            const int cslice = (sp.s0 + j) * kDt;
            const bool rope = ROPE && cslice < p.n_rot;
            if (!kRowPairs && rope) {
                const int c16 = cslice + kCPW * h;
                if (c16 < p.n_rot) {
                    auto unrotate = [&](int r) {
                        const int tok = w.t0() + r;
                        if (tok >= p.T) return;     // zero rows past the sequence's end
                        // pair-major table: a warp's 32 rows read 256 contiguous bytes per pair
                        const float2 *csp = reinterpret_cast<const float2 *>(p.cs) + (size_t)((c16 % p.dh) / 2) * p.T + tok;
                        const uint32_t ra = (uint32_t)r * 128u ^ (((uint32_t)r & 7u) << 4) ^ ((uint32_t)(CH * h) << 4);
                        float2 c[CH * 4];           // every load issued before the first use
#pragma unroll
                        for (int m2 = 0; m2 < CH * 4; ++m2) c[m2] = __ldg(csp + (size_t)m2 * p.T);
                        uint4 u[CH];
#pragma unroll
                        for (int cq = 0; cq < CH; ++cq) u[cq] = lds128(dys + (ra ^ ((uint32_t)cq << 4)));
#pragma unroll
                        for (int cq = 0; cq < CH; ++cq) {
                            float v[8];
                            unpack8(u[cq], v);
#pragma unroll
                            for (int m2 = 0; m2 < 4; ++m2) {
                                const float e0 = v[2 * m2], e1 = v[2 * m2 + 1];
                                const float2 cc = c[4 * cq + m2];
                                v[2 * m2] = fmaf(e0, cc.x, e1 * cc.y);
                                v[2 * m2 + 1] = fmaf(e1, cc.x, -e0 * cc.y);
                            }
                            sts128(dys + (ra ^ ((uint32_t)cq << 4)),
                                   make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]),
                                              pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7])));
                        }
                    };
                    unrotate(row);
                    if (q == 0 && lane < W - 1) unrotate(kTt + lane);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(bar.dyrot());
            }

            // ---- A2: dw[t,g,k] = sum_{c in g} dy[t,c] x[t-k,c], tap-major column k*NG + g.
            // For G < 8 a thread takes one 8-channel chunk (a2c) of two token rows (a2t,
            // a2t+1): one pass over the tile's x rows a2t .. a2t+W serves both rows' W taps
            // (W+3 row loads for two rows instead of 2W+2; lowrank_qkv 0.217 -> 0.210 ms,
            // lowrank_mlp 0.463 -> 0.426 ms).  It reads other threads' dy rows, so with RoPE
            // every warp's rotation is waited for first.  When they fit in registers the
            // values are computed before the dwfree wait: only their stores need the
            // previous tile's dz / dU MMAs to be done with the dw tile.
            constexpr int NPK = (NG8 + 1) / 2;           // packed bf16 pairs per (chunk, tap)
            // (the products of both rows, next to the x window of W+1 rows, in registers)
            constexpr bool kPre = 2 * W * NPK <= 32 && 2 * W * NPK + 4 * (W + 1) <= 52;
            if constexpr (!kRowPairs) {
                // one value per (virtual group, tap): GV = 8 gives one per chunk, and the
                // two chunks' groups are adjacent columns; GV = 16 gives one per warp
                float sv[CH][W];
#pragma unroll
                for (int cq = 0; cq < CH; ++cq) {
                    const uint4 d4 = lds128(dys + (dyr[0] ^ ((uint32_t)cq << 4)));
                    const uint32_t dq[4] = {d4.x, d4.y, d4.z, d4.w};
#pragma unroll
                    for (int k = 0; k < W; ++k) {
                        const uint4 x4 = lds128(xs + (xr[k] ^ ((uint32_t)cq << 4)));
                        const uint32_t xq[4] = {x4.x, x4.y, x4.z, x4.w};
                        float acc = 0.f;
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            acc = (e & 1) ? fma_bf16_hi(dq[e >> 1], xq[e >> 1], acc) : fma_bf16_lo(dq[e >> 1], xq[e >> 1], acc);
                        sv[cq][k] = acc;
                    }
                }
                if (!warp_wait(bar.dwfree(), (i & 1) ^ 1, abort, 32u, &g_fault_bwd, p.wt.wait_ns)) { ok = false; break; }
#pragma unroll
                for (int k = 0; k < W; ++k) {
                    const int jp = k * CL::NB + (GV == 8 ? 2 * h : h);
                    const uint32_t atom = (uint32_t)(jp >> 6), within = (uint32_t)(jp & 63);
                    const uint32_t a = dwrow + atom * 16384u + ((((within >> 3) << 4) ^ dwsw) | ((within & 7) * 2));
                    if constexpr (GV == 8) {
                        sts32(a, pack_bf16x2(sv[0][k], sv[1][k]));
                    } else {
                        const uint32_t pr = pack_bf16x2(sv[0][k] + sv[1][k], 0.f);
                        sts16(a, (uint16_t)(pr & 0xffffu));
                    }
                }
            } else {
                const int ee = ew * 32 + lane;
                const int a2c = ee & 7, a2t = 2 * (ee >> 3);
                auto raddr = [&](int r) {
                    return ((uint32_t)r * 128u) ^ (((uint32_t)r & 7u) << 4) ^ ((uint32_t)a2c << 4);
                };
                uint4 xw[W + 1], d2[2];
#pragma unroll
                for (int ii = 0; ii < 2; ++ii) d2[ii] = lds128(dys + raddr(a2t + ii));
                if (rope) {
                    // rotate this thread's chunk of rows a2t, a2t+1 back (A2 uses the
                    // registers, A1 the copy written back), threads ee < 8(W-1) also one
                    // chunk of a future-halo row; then release A1 (dyrot)
                    const int c8 = cslice + 8 * a2c;
                    if (c8 < p.n_rot) {
                        const float2 *csp = reinterpret_cast<const float2 *>(p.cs) + (size_t)((c8 % p.dh) / 2) * p.T;
                        // every table load is issued before the first use (one round trip)
                        const int tb = w.t0();
                        const bool halo = ee < 8 * (W - 1);
                        const int rh = kTt + (ee >> 3);                 // the halo row, if any
                        const int toks[3] = {tb + a2t, tb + a2t + 1, tb + rh};
                        const bool live[3] = {toks[0] < p.T, toks[1] < p.T, halo && toks[2] < p.T};
                        float2 c[3][4];
#pragma unroll
                        for (int ii = 0; ii < 3; ++ii)
#pragma unroll
                            for (int m2 = 0; m2 < 4; ++m2)
                                c[ii][m2] = live[ii] ? __ldg(csp + (size_t)m2 * p.T + toks[ii]) : make_float2(1.f, 0.f);
                        uint4 uh = make_uint4(0u, 0u, 0u, 0u);
                        if (live[2]) uh = lds128(dys + raddr(rh));
                        auto unrot = [&](uint4 &u, const float2 (&cc)[4]) {
                            float v[8];
                            unpack8(u, v);
#pragma unroll
                            for (int m2 = 0; m2 < 4; ++m2) {
                                const float e0 = v[2 * m2], e1 = v[2 * m2 + 1];
                                v[2 * m2] = fmaf(e0, cc[m2].x, e1 * cc[m2].y);
                                v[2 * m2 + 1] = fmaf(e1, cc[m2].x, -e0 * cc[m2].y);
                            }
                            u = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]),
                                           pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
                        };
                        // rows past the sequence's end stay zero
#pragma unroll
                        for (int ii = 0; ii < 2; ++ii) {
                            if (live[ii]) {
                                unrot(d2[ii], c[ii]);
                                sts128(dys + raddr(a2t + ii), d2[ii]);
                            }
                        }
                        if (live[2]) {
                            unrot(uh, c[2]);
                            sts128(dys + raddr(rh), uh);
                        }
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar.dyrot());
                }
#pragma unroll
                for (int jj = 0; jj <= W; ++jj) xw[jj] = lds128(xs + raddr(a2t + jj));
                // dw of row a2t+ii, tap k: dy row a2t+ii times x tile row a2t+ii+W-1-k
                auto product = [&](int ii, int k, uint32_t (&pk)[NPK]) {
                    const uint4 &d0 = d2[ii];
                    const uint4 &xk = xw[ii + W - 1 - k];
                    if constexpr (G == 1) {
                        // one channel per group: dw = dy * x, exact in fp32 and rounded once
                        // to bf16, which is what the packed bf16 multiply computes
                        pk[0] = bf16x2_mul(d0.x, xk.x);
                        pk[1] = bf16x2_mul(d0.y, xk.y);
                        pk[2] = bf16x2_mul(d0.z, xk.z);
                        pk[3] = bf16x2_mul(d0.w, xk.w);
                    } else {
                        const uint32_t dq[4] = {d0.x, d0.y, d0.z, d0.w};
                        const uint32_t xq[4] = {xk.x, xk.y, xk.z, xk.w};
                        float dwv[NG8];
#pragma unroll
                        for (int gl = 0; gl < NG8; ++gl) {
                            float acc = 0.f;
#pragma unroll
                            for (int e = gl * G; e < (gl + 1) * G; ++e)
                                acc = (e & 1) ? fma_bf16_hi(dq[e >> 1], xq[e >> 1], acc) : fma_bf16_lo(dq[e >> 1], xq[e >> 1], acc);
                            dwv[gl] = acc;
                        }
#pragma unroll
                        for (int m2 = 0; m2 < NG8 / 2; ++m2) pk[m2] = pack_bf16x2(dwv[2 * m2], dwv[2 * m2 + 1]);
                    }
                };
                const int g8 = (8 * a2c) / G;
                auto store = [&](int ii, int k, const uint32_t (&pk)[NPK]) {
                    const uint32_t t = (uint32_t)(a2t + ii);
                    const int jp = k * NGS + g8;                      // first tap-major column
                    const uint32_t atom = (uint32_t)(jp >> 6), within = (uint32_t)(jp & 63);
                    const uint32_t a = sb + p.off_dw + t * 128u + atom * 16384u +
                                       ((((within >> 3) << 4) ^ ((t & 7u) << 4)) | ((within & 7) * 2));
                    if constexpr (NG8 == 8) {
                        sts128(a, make_uint4(pk[0], pk[1], pk[2], pk[3]));
                    } else if constexpr (NG8 == 4) {
                        sts64(a, pk[0], pk[1]);
                    } else {
                        sts32(a, pk[0]);
                    }
                };
                if constexpr (kPre) {
                    uint32_t pk[2][W][NPK];
#pragma unroll
                    for (int ii = 0; ii < 2; ++ii)
#pragma unroll
                        for (int k = 0; k < W; ++k) product(ii, k, pk[ii][k]);
                    if (!warp_wait(bar.dwfree(), (i & 1) ^ 1, abort, 32u, &g_fault_bwd, p.wt.wait_ns)) { ok = false; break; }
#pragma unroll
                    for (int ii = 0; ii < 2; ++ii)
#pragma unroll
                        for (int k = 0; k < W; ++k) store(ii, k, pk[ii][k]);
                } else {
                    if (!warp_wait(bar.dwfree(), (i & 1) ^ 1, abort, 32u, &g_fault_bwd, p.wt.wait_ns)) { ok = false; break; }
#pragma unroll
                    for (int ii = 0; ii < 2; ++ii)
#pragma unroll
                        for (int k = 0; k < W; ++k) {
                            uint32_t pk[NPK];
                            product(ii, k, pk);
                            store(ii, k, pk);
                        }
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(bar.dwready());
                mbar_arrive(bar.xdead());       // this warp's reads of the x tile are done
            }

            // ---- A1: dx[t,c] = dy[t,c] + sum_k w[t+k,g,k] dy[t+k,c]
            if (rope && !warp_wait(bar.dyrot(), (nrot++) & 1, abort, 8192u, &g_fault_bwd, p.wt.wait_ns)) { ok = false; break; }
            if (!warp_wait(bar.wfull(), i & 1, abort, 128u, &g_fault_bwd, p.wt.wait_ns)) { ok = false; break; }
            tc_fence_after();
            constexpr int NGB = NG8;                        // (virtual) groups of one chunk
            constexpr int KB = (W * (4 + NGB) <= 48) ? W : 4;   // taps per batch
            uint4 dxo[CH];
#pragma unroll
            for (int cq = 0; cq < CH; ++cq) {
                float dx[8];
                uint64_t acc[4];
#pragma unroll
                for (int k0 = 0; k0 < W; k0 += KB) {
                    uint4 du[KB];
                    uint32_t wr[KB][NGB];
#pragma unroll
                    for (int kb = 0; kb < KB; ++kb)
                        if (k0 + kb < W) du[kb] = lds128(dys + (dyr[k0 + kb] ^ ((uint32_t)cq << 4)));
#pragma unroll
                    for (int kb = 0; kb < KB; ++kb)
                        if (k0 + kb < W)
                            tmem_ld<NGB>(tl + p.tm_w + (k0 + kb) * CL::NB + (kCPW * h + 8 * cq) / GV, wr[kb]);
                    tmem_wait_ld();
#pragma unroll
                    for (int kb = 0; kb < KB; ++kb)
#pragma unroll
                        for (int e = 0; e < NGB; ++e) asm volatile("" : "+r"(wr[kb][e]));
#pragma unroll
                    for (int kb = 0; kb < KB; ++kb) {
                        const int k = k0 + kb;
                        if (k >= W) break;
                        if constexpr (G == 1) {
                            // channel pairs in packed fp32 FMAs (the same roundings as scalar fmaf)
                            const uint32_t u[4] = {du[kb].x, du[kb].y, du[kb].z, du[kb].w};
#pragma unroll
                            for (int m = 0; m < 4; ++m) {
                                const uint64_t d2 = f2pack(bf16_lo(u[m]), bf16_hi(u[m]));
                                const uint64_t w2 = f2pack(__uint_as_float(wr[kb][2 * m]), __uint_as_float(wr[kb][2 * m + 1]));
                                acc[m] = f2fma(w2, d2, k == 0 ? d2 : acc[m]);
                            }
                        } else {
                            float dk[8];
                            unpack8(du[kb], dk);
#pragma unroll
                            for (int e = 0; e < 8; ++e)
                                dx[e] = fmaf(__uint_as_float(wr[kb][e / GV]), dk[e], k == 0 ? dk[e] : dx[e]);
                        }
                    }
                }
                if constexpr (G == 1) {
#pragma unroll
                    for (int m = 0; m < 4; ++m) f2unpack(acc[m], dx[2 * m], dx[2 * m + 1]);
                }
                dxo[cq].x = pack_bf16x2(dx[0], dx[1]);
                dxo[cq].y = pack_bf16x2(dx[2], dx[3]);
                dxo[cq].z = pack_bf16x2(dx[4], dx[5]);
                dxo[cq].w = pack_bf16x2(dx[6], dx[7]);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar.wempty());
            // once every epilogue warp is past A2 the x tile is dead, and dx goes there
            // (an mbarrier rather than a named barrier, so that the wait is bounded)
            if (!warp_wait(bar.xdead(), i & 1, abort, 4096u, &g_fault_bwd, p.wt.wait_ns)) { ok = false; break; }
#pragma unroll
            for (int cq = 0; cq < CH; ++cq) sts128(xs + (dxr0 ^ ((uint32_t)cq << 4)), dxo[cq]);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar.dxr(st));

            // ---- dz of the previous token tile, complete once its last slice's MMAs ran
            // the previous token tile's dz; half the warps a slice later, so that fewer
            // reductions queue at once (lowrank_qkv 0.238 -> 0.227 ms)
            {
                const int jd = (S >= 2 && h >= 2) ? 1 : 0;
                if (j == jd && mz > 0 && !dz_out(mz - 1, pb, pt0)) { ok = false; break; }
            }
            if (j == S - 1) {
                pb = w.b;
                pt0 = w.t0();
            }
        }
        if (ok && nt > 0) ok = dz_out(nt / S - 1, pb, pt0);

        // ---- dU: this CTA's partial of each of its slices, then the slice group's sum
        if (ok && warp_wait(bar.dufull(), 0, abort, 512u, &g_fault_bwd, p.wt.wait_ns)) {
            tc_fence_after();
            const int N = p.n_slices * p.SC;
            for (int j = 0; j < S; ++j) {
                const int slice = sp.s0 + j;
                if (h < CL::NMB) {
                    // lane j' of dU^T M-block h is tap-major column k*NB + gv; the real
                    // column of U is g*W + k with g the (virtual) group's real group
                    const int jp = 128 * h + row;
                    const int k = jp / CL::NB, gv = jp % CL::NB;
                    const bool valid = k < W && gv < CL::NGV && gv % CL::VPR == 0;
                    const int jn = (gv * GV / G) * W + k;
                    float *dst = p.du_part + (size_t)sp.a * p.R * N + (size_t)slice * p.SC + jn;
#pragma unroll 1
                    for (int c0 = 0; c0 < p.R; c0 += 16) {
                        uint32_t v[16];
                        tmem_ld<16>(tl + p.tm_du + (j * CL::NMB + h) * p.R + c0, v);   // warp-collective
                        tmem_wait_ld_regs(v);
                        float f[16];
#pragma unroll
                        for (int m2 = 0; m2 < 16; ++m2) f[m2] = __uint_as_float(v[m2]);
                        if constexpr (CL::VPR >= 2) {
#pragma unroll
                            for (int m2 = 0; m2 < 16; ++m2) f[m2] += __shfl_xor_sync(0xffffffffu, f[m2], 1);
                        }
                        if constexpr (CL::VPR >= 4) {
#pragma unroll
                            for (int m2 = 0; m2 < 16; ++m2) f[m2] += __shfl_xor_sync(0xffffffffu, f[m2], 2);
                        }
                        if (valid) {
#pragma unroll
                            for (int m2 = 0; m2 < 16; ++m2) dst[(size_t)(c0 + m2) * N] = f[m2];
                        }
                    }
                }
            }
            tc_fence_before();
            fence_gpu();
            __syncwarp();
            if (lane == 0) red_release_add(p.flag_du + sp.b, 1u);
            if (wait_count(p.flag_du + sp.b, (unsigned)(kEpiWarps * p.A), abort, 1024u, p.wt.wait_ns)) {
                // this CTA's share (of A) of the group's R x (S*SC) block
                const int cols = S * p.SC;
                const long long n = (long long)p.R * cols;
                const long long e0 = n * sp.a / p.A, e1 = n * (sp.a + 1) / p.A;
                const int et = threadIdx.x - 32 * kEpi0;
                for (long long e = e0 + et; e < e1; e += 32 * kEpiWarps) {
                    const int r = (int)(e / cols), c = (int)(e - (long long)r * cols);
                    const size_t off = (size_t)r * N + (size_t)sp.s0 * p.SC + c;
                    float acc = 0.f;
                    for (int a = 0; a < p.A; ++a) acc += __ldcg(p.du_part + (size_t)a * p.R * N + off);
                    p.dU[off] = acc;
                }
            }
        }
        __syncwarp();
    } else if (warp == kMmaWarp) {
        // ---------------------------------------------------------- MMA issuer: dz and dU
        // Once tile i's dw is written:
        //   dz[m] (+)= dw Up^T: A = dw tile (K-major view), B = Up slice (K-major), 16
        //     columns per step (+32 bytes within a 64-column atom, the next atom every 4
        //     steps); accumulates over the token tile's slices;
        //   dU^T[slice] (+)= dw^T z: A = dw^T (MN-major), B = z tile rows 0..127
        //     (MN-major), 16 tokens per step; accumulates over the CTA's token tiles.
        // The step counts are compile-time, so the issue loops unroll fully.
        constexpr int KSC = CL::SCQ / 16;
        constexpr int NMB = CL::NMB;
        const uint64_t t_k128 = desc_tmpl(16, 1024, kSw128);
        const uint64_t t_dwt = desc_tmpl(16384, 1024, kSw128);
        const uint64_t t_zmn = desc_tmpl(128, p.z_slab, kSwNone);
        const uint32_t i_dz = idesc_bf16(128, p.R, false, false);
        const uint32_t i_du = idesc_bf16(128, p.R, true, true);
        const uint32_t ubox = (uint32_t)(p.R * 128);
        const uint64_t st_wrap_a = (16384u - 96u) >> 4;   // next 64-column dw atom
        const uint64_t st_wrap_b = (ubox - 96u) >> 4;     // next 64-column Up box
        const uint32_t dw0 = sb + p.off_dw;
        for (Walk w(sp.m0, p.tiles_per_seq); w.i < nt; w.next(S, NST, p.tiles_per_seq)) {
            const int i = w.i, j = w.j, mz = w.mz, db = mz & 1, zb = mz & 1;
            const int ub = u_res ? j : (i & 1);
            const int upar = u_res ? 0 : ((i >> 1) & 1);
            if (!warp_wait(bar.ufull(ub), upar, abort, 4u, &g_fault_bwd, p.wt.wait_ns)) break;
            if (j == 0 && !warp_wait(bar.zfull(zb), (mz >> 1) & 1, abort, 4u, &g_fault_bwd, p.wt.wait_ns)) break;
            if (!warp_wait(bar.dwready(), i & 1, abort, 8u, &g_fault_bwd, p.wt.wait_ns)) break;
            if (j == 0 && !warp_wait(bar.dzempty(db), ((mz >> 1) & 1) ^ 1, abort, 8u, &g_fault_bwd, p.wt.wait_ns)) break;
            tc_fence_after();
            if (elect_one()) {      // one lane issues the tile's MMAs and commits
                {
                    const uint32_t us = sb + p.off_u + ub * p.u_bytes;
                    uint64_t da = desc_at(t_k128, dw0), dbd = desc_at(t_k128, us);
                    const uint32_t d = tmem + p.tm_dz + db * p.R;
#pragma unroll
                    for (int kk = 0; kk < KSC; ++kk) {
                        mma_bf16_ss(d, da, dbd, i_dz, (j > 0 || kk > 0) ? 1u : 0u);
                        const bool wrap = (kk & 3) == 3;
                        da += wrap ? st_wrap_a : 2u;
                        dbd += wrap ? st_wrap_b : 2u;
                    }
                }
                {
                    const uint32_t zs = sb + p.off_z + zb * p.z_bytes;
#pragma unroll
                    for (int mb = 0; mb < NMB; ++mb) {
                        const uint32_t d = tmem + p.tm_du + (j * NMB + mb) * p.R;
                        uint64_t da = desc_at(t_dwt, dw0 + mb * 32768u), dbd = desc_at(t_zmn, zs);
#pragma unroll
                        for (int kk = 0; kk < kTt / 16; ++kk) {
                            mma_bf16_ss(d, da, dbd, i_du, (mz == 0 && kk == 0) ? 0u : 1u);
                            da += 2048u >> 4;
                            dbd += 256u >> 4;
                        }
                    }
                }
                mma_commit(bar.dwfree());
                if (!u_res) mma_commit(bar.uempty(ub));
                if (j == S - 1) {
                    mma_commit(bar.dzfull(db));
                    mma_commit(bar.zempty(zb));
                }
            }
            __syncwarp();
        }
        if (elect_one()) {
            mma_commit(bar.dufull());
            mma_commit(bar.done());
        }
        __syncwarp();
    }

    __syncthreads();
    if (warp == kRecWarp) {
        if (lane == 0) mbar_drain(bar.done(), 0, p.wt.wait_ns);
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, p.tmem_cols);
    }
}

// Up[r, s*SCq + k*NB + gv] = U[r, (real group of virtual group gv of slice s)*W + k], and
// 0 for padding columns gv >= NGV (see Cols).  For G <= 4 that is the tap-major
// reordering Up[r, s*SC + k*NG + g] = U[r, s*SC + g*W + k].
// Grid (ceil(N'/2048), R): one row r per grid row; each thread writes 8 consecutive output
// columns (one tap, 8 consecutive (virtual) groups) with one 16-byte store.  Block (0, 0)
// also clears the main kernel's counters, and all threads zero dz (which the main
// kernel adds into).
__global__ void k_permute_u(const bf16 *__restrict__ U, bf16 *__restrict__ Up, int R, int N, int Nq, int SCq,
                            int NB, int NGV, int GV, int G, int W, unsigned *__restrict__ flags, int nflags,
                            float4 *__restrict__ dz, long long ndz4) {
    if (blockIdx.x == 0 && blockIdx.y == 0)
        for (int f = threadIdx.x; f < nflags; f += blockDim.x) flags[f] = 0u;
    {
        // dz is summed into by the main kernel: start it at zero
        const long long nth = (long long)gridDim.x * gridDim.y * blockDim.x;
        const long long id = ((long long)blockIdx.y * gridDim.x + blockIdx.x) * blockDim.x + threadIdx.x;
        for (long long e = id; e < ndz4; e += nth) dz[e] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    const int r = blockIdx.y;
    const int j = 8 * (blockIdx.x * blockDim.x + threadIdx.x);
    if (r >= R || j >= Nq) return;
    const int s = j / SCq, jl = j - s * SCq;
    const int k = jl / NB, gv0 = jl - k * NB;
    const unsigned short *src = reinterpret_cast<const unsigned short *>(U) + (size_t)r * N;
    uint32_t v[4];
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        uint32_t h2[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int gv = gv0 + 2 * m + e;
            h2[e] = gv < NGV ? (uint32_t)src[(size_t)((s * 64 + gv * GV) / G) * W + k] : 0u;
        }
        v[m] = h2[0] | (h2[1] << 16);
    }
    *reinterpret_cast<uint4 *>(Up + (size_t)r * Nq + j) = make_uint4(v[0], v[1], v[2], v[3]);
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

bool make_map(CUtensorMap *m, const void *ptr, int rank, const uint64_t *dims, const uint32_t *box,
              CUtensorMapSwizzle sw, CUtensorMapL2promotion promo) {
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
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void *>(ptr), gdim, gstride, bdim, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, sw, promo, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int num_sms() {
    static int n[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return 148;
    if (!n[dev]) cudaDeviceGetAttribute(&n[dev], cudaDevAttrMultiProcessorCount, dev);
    return n[dev] > 0 ? n[dev] : 148;
}

constexpr uint32_t kSmemLimit = 227 * 1024;
size_t a256(size_t v) { return (v + 255) / 256 * 256; }
uint32_t a1k(uint32_t v) { return (v + 1023) / 1024 * 1024; }

uint32_t smem_bytes(const BwdParams &p) { return p.off_bar + kBarBytes + 16 + 1024; }

// Shared-memory layout for a ring depth and number of Up buffers; false if it does not fit.
bool layout_smem(BwdParams &p, int stages, int nU) {
    p.stages = stages;
    p.nU = nU;
    p.off_z = stages * p.stage_bytes;
    p.off_u = p.off_z + 2 * p.z_bytes;
    p.off_dw = a1k(p.off_u + nU * p.u_bytes);
    p.off_bar = p.off_dw + (uint32_t)(p.SCp / 64) * 16384u;
    return smem_bytes(p) <= kSmemLimit;
}

// Plans the kernel for these sizes on `nsm` SMs: tile geometry, TMEM and shared-memory
// layouts, and the A x Bg grid.  false: the tensor-core backward does not take them.
bool plan_bwd(int B, int T, int D, int G, int W, int R, int nsm, BwdParams &p) {
    if (!(R == 16 || R == 32 || R == 64)) return false;
    if (D % kDt || !(G == 1 || G == 2 || G == 4 || G == 8 || G == 16 || G == 32 || G == 64) || W < 1 || W > 8)
        return false;
    p = BwdParams{};
    p.B = B; p.T = T; p.D = D; p.G = G; p.W = W; p.R = R;
    p.NGs = kDt / G;
    const int gv = G < 16 ? G : 16;                   // mirrors Cols<W, G>
    p.NGp = (kDt / gv) < 16 ? 16 : kDt / gv;
    p.SC = p.NGs * W;
    p.SCq = p.NGp * W;
    if (p.SCq % 16) return false;
    p.SCp = (p.SCq + 127) / 128 * 128;
    p.n_slices = D / kDt;
    p.tiles_per_seq = (T + kTt - 1) / kTt;
    const long long ntt = (long long)B * p.tiles_per_seq;
    if (ntt >= (1ll << 30) || (long long)p.n_slices * ntt >= (1ll << 31)) return false;
    p.n_tt = (int)ntt;
    p.u_boxes = (p.SCq + 63) / 64;
    // TMEM: w (W tap blocks) | dz (two buffers) | dU^T (one slot per slice of the CTA)
    p.tm_w = 0;
    p.tm_dz = (uint32_t)(W * p.NGp + 31) / 32 * 32;
    p.tm_du = p.tm_dz + 2u * (uint32_t)R;
    const uint32_t slot = (uint32_t)(p.SCp / 128) * R;
    if (p.tm_du + slot > 512) return false;
    const int s_max_tmem = (int)((512 - p.tm_du) / slot);
    // shared memory
    p.rows = kTt + W - 1;
    p.xy_tile_bytes = a1k(p.rows * 128);
    p.z_slab = (p.rows * 16 + 127) / 128 * 128;
    p.z_bytes = a1k((uint32_t)(R / 8) * p.z_slab);
    p.stage_bytes = 2 * p.xy_tile_bytes;
    p.u_bytes = (uint32_t)(p.u_boxes * R * 128);
    // grid: Bg slice groups (at most s_max_tmem slices each) x A token ranges; fewest
    // tiles on the busiest CTA first, then fewest slice groups (fewer dz partials)
    int best_bg = 0, best_a = 0;
    long long best_cost = -1;
    for (int bg = 1; bg <= std::min(p.n_slices, nsm); ++bg) {
        const int smax = (p.n_slices + bg - 1) / bg;
        if (smax > s_max_tmem) continue;
        const int a = std::min(p.n_tt, nsm / bg);
        if (a < 1) continue;
        const long long cost = (long long)smax * ((p.n_tt + a - 1) / a);
        if (best_cost < 0 || cost < best_cost) {
            best_cost = cost;
            best_bg = bg;
            best_a = a;
        }
    }
    if (best_cost < 0) return false;
    p.Bg = best_bg;
    p.A = best_a;
    const int smax = (p.n_slices + p.Bg - 1) / p.Bg;
    p.tmem_cols = 32;
    while (p.tmem_cols < p.tm_du + (uint32_t)smax * slot) p.tmem_cols *= 2;
    // ring depth 3 if it fits, else 2; two Up buffers unless a CTA has one slice
    const int nU = smax >= 2 ? 2 : 1;
    for (int st = kMaxStages; st >= 2; --st)
        if (layout_smem(p, st, nU)) return true;
    return false;
}

template <int W, int G>
cudaError_t launch_t(const CUtensorMap *m, const BwdParams &p, cudaStream_t s) {
    auto kern = p.n_rot > 0 ? k_tc_lowrank_bwd<W, G, true> : k_tc_lowrank_bwd<W, G, false>;
    const uint32_t smem = smem_bytes(p);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    // Cooperative launch: the CTAs wait on each other's partial sums, so all of them
    // must be resident at once (the launch fails instead of starting otherwise).
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.A * p.Bg);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, m[0], m[1], m[2], m[3], m[4], p);
}

template <int W>
cudaError_t launch_w(int G, const CUtensorMap *m, const BwdParams &p, cudaStream_t s) {
    switch (G) {
        case 1: return launch_t<W, 1>(m, p, s);
        case 2: return launch_t<W, 2>(m, p, s);
        case 4: return launch_t<W, 4>(m, p, s);
        case 8: return launch_t<W, 8>(m, p, s);
        case 16: return launch_t<W, 16>(m, p, s);
        case 32: return launch_t<W, 32>(m, p, s);
        default: return launch_t<W, 64>(m, p, s);
    }
}

struct WsLayout {
    size_t up, du, flags, total;
};

WsLayout ws_layout(const BwdParams &p) {
    WsLayout l;
    const size_t N = (size_t)p.n_slices * p.SC;
    const size_t Nq = (size_t)p.n_slices * p.SCq;
    l.up = 0;
    l.du = a256(l.up + (size_t)p.R * Nq * 2);
    l.flags = a256(l.du + (size_t)p.A * p.R * N * 4);
    l.total = a256(l.flags + (size_t)p.Bg * 4);
    return l;
}

}  // namespace
}  // namespace tcb

bool tc_lowrank_bwd_supported(int B, int T, int D, int G, int W, int R, bool bf16) {
    tcb::BwdParams p;
    return bf16 && tcb::plan_bwd(B, T, D, G, W, R, tcb::num_sms(), p);
}

size_t tc_lowrank_bwd_workspace(int B, int T, int D, int G, int W, int R) {
    tcb::BwdParams p;
    if (!tcb::plan_bwd(B, T, D, G, W, R, tcb::num_sms(), p)) return 0;
    return tcb::ws_layout(p).total;
}

cudaError_t launch_tc_lowrank_bwd(const void *x, const void *z, const void *U, const void *dy, void *dx,
                                  float *dz, float *dU, void *ws, int B, int T, int D, int G, int W, int R,
                                  cudaStream_t s, const float *cs, int dh, int n_rot) {
    using namespace tcb;
    BwdParams p;
    if (!plan_bwd(B, T, D, G, W, R, num_sms(), p)) return cudaErrorNotSupported;
    p.cs = cs;
    p.dh = dh;
    p.n_rot = cs ? n_rot : 0;
    take_wait_test(&p.wt.wait_ns, &p.wt.withhold_cta);
    const WsLayout l = ws_layout(p);
    uint8_t *w8 = (uint8_t *)ws;
    bf16 *Up = (bf16 *)(w8 + l.up);
    p.du_part = (float *)(w8 + l.du);
    p.flag_du = (unsigned *)(w8 + l.flags);
    p.dz = dz;
    p.dU = dU;
    const int N = p.n_slices * p.SC;
    const int Nq = p.n_slices * p.SCq;
    const int gv = G < 16 ? G : 16;
    k_permute_u<<<dim3((Nq / 8 + 255) / 256, R), 256, 0, s>>>((const bf16 *)U, Up, R, N, Nq, p.SCq, p.NGp,
                                                               kDt / gv, gv, G, W, p.flag_du, p.Bg,
                                                               (float4 *)dz, (long long)B * T * R / 4);

    CUtensorMap m[5];
    const uint64_t dxyz[3] = {(uint64_t)D, (uint64_t)T, (uint64_t)B};
    const uint32_t bxy[3] = {(uint32_t)kDt, p.rows, 1};
    const uint64_t dzz[3] = {(uint64_t)R, (uint64_t)T, (uint64_t)B};
    const uint32_t bz[3] = {8, p.rows, 1};
    const uint64_t du[2] = {(uint64_t)Nq, (uint64_t)R};
    const uint32_t bu[2] = {64, (uint32_t)R};
    const uint32_t bdx[3] = {(uint32_t)kDt, (uint32_t)kTt, 1};
    if (!make_map(&m[0], dy, 3, dxyz, bxy, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B) ||
        !make_map(&m[1], x, 3, dxyz, bxy, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B) ||
        !make_map(&m[2], z, 3, dzz, bz, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B) ||
        !make_map(&m[3], Up, 2, du, bu, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B) ||
        !make_map(&m[4], dx, 3, dxyz, bdx, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B)) {
        set_last_error("dsc_bwd_lowrank: cuTensorMapEncodeTiled failed");
        return cudaErrorInvalidValue;
    }
    switch (W) {
        case 1: return launch_w<1>(G, m, p, s);
        case 2: return launch_w<2>(G, m, p, s);
        case 3: return launch_w<3>(G, m, p, s);
        case 4: return launch_w<4>(G, m, p, s);
        case 5: return launch_w<5>(G, m, p, s);
        case 6: return launch_w<6>(G, m, p, s);
        case 7: return launch_w<7>(G, m, p, s);
        default: return launch_w<8>(G, m, p, s);
    }
}

unsigned read_device_fault_bwd(bool reset) {
    unsigned v = 0;
    if (cudaMemcpyFromSymbol(&v, tcb::g_fault_bwd, sizeof(v)) != cudaSuccess) return 0xffffffffu;
    if (reset) {
        const unsigned zero = 0;
        cudaMemcpyToSymbol(tcb::g_fault_bwd, &zero, sizeof(zero));
    }
    return v;
}

}  // namespace dsc
