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
// W/G times the bytes of x).
//
// Work tile = 128 tokens of one sequence x one 64-channel slice.  Per tile:
//   1. recompute, one MMA per tap k with the z tile shifted by k rows:
//        Wk[t, g] = sum_r z[t0+t+k, r] Up[r, k*NG+g]   (Up: U with the slice's columns
//      reordered tap-major by a pre-pass), so TMEM lane t holds w[t+k, g, k] for every k;
//   2. epilogue (one token row per thread): dx and dw on CUDA cores; dx is stored by TMA,
//      dw (bf16) is written to shared memory;
//   3. dz partial = dw Up^T   (A = dw tile, B = Up slice, M=128 tokens, N=R);
//      dU^T     += dw^T z     (A = the same tile read MN-major, B = z tile, M=128 columns,
//      N=R), accumulated in TMEM over all tiles of the slice that the CTA processes.
//   Recompute, dz and dU are issued by three MMA warps, each on its own SM sub-partition.
// Persistent CTAs own contiguous tile ranges in slice-major order.  dz partials (per
// slice) and dU partials (per CTA segment of a slice) go to the workspace and are summed
// in a fixed order by one small kernel, so results are deterministic.
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
// Epilogue geometry: 16 warps of 16 channels (4 TMEM lane quarters x 4 channel groups).
// (8 warps of 32 channels, with 168 registers a thread, measured slower at G=4, W=8:
// 0.76 against 0.74 ms on the lowrank_mlp backward.)
// Warp roles: 0 TMA producer, 1 recompute MMAs, 2..1+E epilogue, 2+E dz MMAs, 3+E dU MMAs.
// The three MMA streams are issued from warps on three different SM sub-partitions: one
// warp issuing all of them shares its issue slots with the busy epilogue warps and cannot
// keep the tensor pipe fed.
template <int G>
struct Geo {
    static constexpr int kEpiWarps = 16;
    static constexpr int kGroups = kEpiWarps / 4;      // channel groups of a slice
    static constexpr int kCPW = kDt / kGroups;         // channels per epilogue warp
    static constexpr int kDxBuf = 32 * kCPW * 2;       // one warp's dx staging: 32 rows x kCPW bf16
    static constexpr int kDzWarp = 2 + kEpiWarps;
    static constexpr int kDuWarp = 3 + kEpiWarps;
    static constexpr int kThreads = 32 * (4 + kEpiWarps);
};
constexpr uint32_t kDxStageBytes = 4 * 32 * kDt * 2;   // all epilogue warps' dx staging

struct BwdParams {
    int B, T, D, G, W, R;
    int NGs;                  // filter groups per slice (64/G)
    int NGp;                  // TMEM columns per tap block (NGs rounded up to 16)
    int SC;                   // filter columns per slice (NGs*W)
    int SCp;                  // SC rounded up to 128 (dU^T M-blocks)
    int n_slices, tiles_per_seq, per_slice, n_tiles, maxseg;
    int u_boxes;              // TMA boxes of 64 Up columns per slice
    int nU, stages;
    uint32_t rows;            // tile rows incl. halo: 128 + W - 1
    uint32_t xy_tile_bytes;   // one dy or x tile (rows x 128 B), 1024-aligned
    uint32_t z_slab;          // stride of the 8-wide z slabs (rows x 16 B, rounded up to 128:
                              // a TMA destination must be 128-byte aligned)
    uint32_t z_bytes;         // R/8 slabs
    uint32_t u_bytes;
    uint32_t stage_bytes;     // dy tile + x tile + z tile
    uint32_t off_u, off_dw, off_dx, off_bar;
    uint32_t tm_w, tm_dw, tm_dz, tm_du, tmem_cols;   // TMEM column map
    float *dz_part;           // [n_slices][B*T][R]
    float *du_part;           // [n_slices][maxseg][R][SC]
};

struct Bars {
    uint32_t base;
    __device__ uint32_t full(int s) const { return base + 8 * s; }
    __device__ uint32_t empty(int s) const { return base + 8 * (3 + s); }
    __device__ uint32_t uf(int u) const { return base + 8 * (6 + u); }
    __device__ uint32_t ue(int u) const { return base + 8 * (8 + u); }
    __device__ uint32_t wfull() const { return base + 8 * 10; }
    __device__ uint32_t wempty() const { return base + 8 * 11; }
    __device__ uint32_t dwready() const { return base + 8 * 12; }
    __device__ uint32_t mm2() const { return base + 8 * 13; }
    __device__ uint32_t done() const { return base + 8 * 14; }
};
constexpr uint32_t kBarBytes = 8 * 15;

__device__ __forceinline__ void unpack8(const uint4 &u, float (&v)[8]) {
    v[0] = bf16_lo(u.x); v[1] = bf16_hi(u.x);
    v[2] = bf16_lo(u.y); v[3] = bf16_hi(u.y);
    v[4] = bf16_lo(u.z); v[5] = bf16_hi(u.z);
    v[6] = bf16_lo(u.w); v[7] = bf16_hi(u.w);
}

template <int N> __device__ __forceinline__ void tmem_st_n(uint32_t a, const uint32_t *r);
template <> __device__ __forceinline__ void tmem_st_n<1>(uint32_t a, const uint32_t *r) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x1.b32 [%0], {%1};" ::"r"(a), "r"(r[0]) : "memory");
}
template <> __device__ __forceinline__ void tmem_st_n<2>(uint32_t a, const uint32_t *r) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x2.b32 [%0], {%1, %2};" ::"r"(a), "r"(r[0]), "r"(r[1])
                 : "memory");
}
template <> __device__ __forceinline__ void tmem_st_n<4>(uint32_t a, const uint32_t *r) { tmem_st<4>(a, r); }

__device__ __forceinline__ void sts32(uint32_t addr, uint32_t v) {
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ void sts64(uint32_t addr, uint32_t a, uint32_t b) {
    asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(addr), "r"(a), "r"(b) : "memory");
}

// Tile index -> (slice, sequence, first token)
struct TileId {
    int slice, b, t0;
};
__device__ __forceinline__ TileId tile_id(const BwdParams &p, int i) {
    TileId id;
    id.slice = i / p.per_slice;
    const int rem = i - id.slice * p.per_slice;
    id.b = rem / p.tiles_per_seq;
    id.t0 = (rem - id.b * p.tiles_per_seq) * kTt;
    return id;
}

// CTA that owns tile i when n tiles are split into contiguous ranges over g CTAs
// (CTA c owns [c*n/g, (c+1)*n/g)).
__host__ __device__ inline int owner_of(long long i, long long n, long long g) {
    return (int)(((i + 1) * g - 1) / n);
}

template <int W, int G>
__global__ void __launch_bounds__(Geo<G>::kThreads, 1)
k_tc_lowrank_bwd(const __grid_constant__ CUtensorMap tm_dy, const __grid_constant__ CUtensorMap tm_x,
                 const __grid_constant__ CUtensorMap tm_z, const __grid_constant__ CUtensorMap tm_u,
                 const __grid_constant__ CUtensorMap tm_dx, const BwdParams p) {
    constexpr int NG8 = 8 / G;          // filter groups in one 8-channel chunk
    constexpr int kEpiWarps = Geo<G>::kEpiWarps, kCPW = Geo<G>::kCPW, kDxBuf = Geo<G>::kDxBuf;
    constexpr int kDzWarp = Geo<G>::kDzWarp, kDuWarp = Geo<G>::kDuWarp, kThreads = Geo<G>::kThreads;
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
            mbar_init(bar.empty(s), kEpiWarps);
        }
        for (int u = 0; u < 2; ++u) {
            mbar_init(bar.uf(u), 1);
            mbar_init(bar.ue(u), 2);        // recompute and dz streams
        }
        mbar_init(bar.wfull(), 1);
        mbar_init(bar.wempty(), kEpiWarps);
        mbar_init(bar.dwready(), kEpiWarps);
        mbar_init(bar.mm2(), 2);            // dz and dU streams
        mbar_init(bar.done(), 3);           // all three MMA streams
        *abort = 0;
        fence_barrier_init();
    }
    // dw^T rows beyond SC (padding of the last 128-column M-block) must read as zero.
    if (p.SCp > p.SC) {
        for (uint32_t o = threadIdx.x * 16; o < (uint32_t)(p.SCp / 64) * 16384u; o += kThreads * 16) {
            const uint32_t atom = o / 16384u;
            if ((int)(atom * 64) + 64 > p.SC) sts128(sb + p.off_dw + o, make_uint4(0, 0, 0, 0));
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
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_holder), p.tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    const int tbeg = (int)((long long)blockIdx.x * p.n_tiles / gridDim.x);
    const int tend = (int)((long long)(blockIdx.x + 1) * p.n_tiles / gridDim.x);

    if (warp == 0) {
        // ---------------------------------------------------------- TMA producer
        if (lane == 0) {
            int prev = -1, v = -1;
            const uint32_t tx = 2 * p.rows * 128 + (uint32_t)(p.R / 8) * p.rows * 16;   // bytes TMA delivers
            for (int i = tbeg; i < tend; ++i) {
                const int it = i - tbeg;
                const TileId id = tile_id(p, i);
                if (id.slice != prev) {
                    prev = id.slice;
                    ++v;
                    const int ub = v % p.nU, un = v / p.nU;
                    if (!mbar_wait(bar.ue(ub), (un & 1) ^ 1, abort, 1u, &g_fault_bwd)) break;
                    mbar_arrive_expect_tx(bar.uf(ub), p.u_bytes);
                    const uint32_t ud = sb + p.off_u + ub * p.u_bytes;
                    for (int bx = 0; bx < p.u_boxes; ++bx)
                        tma_load_2d(ud + bx * (uint32_t)(p.R * 128), &tm_u, bar.uf(ub),
                                    id.slice * p.SC + 64 * bx, 0);
                }
                const int s = it % p.stages, n = it / p.stages;
                if (!mbar_wait(bar.empty(s), (n & 1) ^ 1, abort, 2u, &g_fault_bwd)) break;
                mbar_arrive_expect_tx(bar.full(s), tx);
                const uint32_t st = sb + s * p.stage_bytes;
                tma_load_3d(st, &tm_dy, bar.full(s), id.slice * kDt, id.t0, id.b);
                tma_load_3d(st + p.xy_tile_bytes, &tm_x, bar.full(s), id.slice * kDt, id.t0 - (W - 1), id.b);
                for (int j = 0; j < p.R / 8; ++j)
                    tma_load_3d(st + 2 * p.xy_tile_bytes + j * p.z_slab, &tm_z, bar.full(s), 8 * j, id.t0, id.b);
            }
            const int issued = tend - tbeg;
            for (int s = 0; s < p.stages && s < issued; ++s) {
                const int last = issued - 1 - ((issued - 1 - s) % p.stages);
                mbar_wait(bar.full(s), (last / p.stages) & 1, abort, 0u, &g_fault_bwd);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer: recompute
        // Each MMA warp runs its schedule warp-uniformly; one elected lane issues each
        // tcgen05 instruction, and descriptors advance by adding to their start field.
        // Tile i's filters are recomputed once the epilogue has read those of tile i-1.
        const uint64_t t_zk = desc_tmpl(p.z_slab, 128, kSwNone);               // z, K-major, no swizzle
        const uint64_t t_u_mn = desc_tmpl((uint32_t)(p.R * 128), 1024, kSw128);  // Up as MN-major B
        const uint32_t i_rec = idesc_bf16(128, p.NGp, false, true);
        const int ksr = p.R / 16;
        const uint32_t ubox = (uint32_t)(p.R * 128);
        const uint64_t st_zk = (2 * p.z_slab) >> 4;   // 16 more z columns (start field units)
        int prev_slice = -1, v = -1, ub = 0;
        for (int i = tbeg; i < tend; ++i) {
            const int it = i - tbeg;
            const TileId id = tile_id(p, i);
            if (id.slice != prev_slice) {
                prev_slice = id.slice;
                ++v;
                ub = v % p.nU;
                if (!warp_wait(bar.uf(ub), (v / p.nU) & 1, abort, 4u, &g_fault_bwd)) break;
            }
            const int s = it % p.stages, n = it / p.stages;
            if (!warp_wait(bar.full(s), n & 1, abort, 8u, &g_fault_bwd)) break;
            if (!warp_wait(bar.wempty(), (it & 1) ^ 1, abort, 16u, &g_fault_bwd)) break;
            tc_fence_after();
            const uint32_t zs = sb + s * p.stage_bytes + 2 * p.xy_tile_bytes;
            const uint32_t us = sb + p.off_u + ub * p.u_bytes;
#pragma unroll
            for (int k = 0; k < W; ++k) {
                const int col0 = k * (kDt / G);
                uint64_t da = desc_at(t_zk, zs + 16 * k);
                uint64_t db = desc_at(t_u_mn, us + (col0 / 64) * ubox + (col0 % 64) * 2);
                const uint32_t d = tmem + p.tm_w + k * p.NGp;
                for (int kk = 0; kk < ksr; ++kk) {
                    if (elect_one()) mma_bf16_ss(d, da, db, i_rec, kk > 0 ? 1u : 0u);
                    __syncwarp();
                    da += st_zk;
                    db += 2048u >> 4;
                }
            }
            const bool last_of_slice = (i + 1 == tend) || ((i + 1) / p.per_slice != id.slice);
            if (elect_one()) {
                mma_commit(bar.wfull());
                if (last_of_slice) mma_commit(bar.ue(ub));
            }
            __syncwarp();
        }
        if (elect_one()) mma_commit(bar.done());
        __syncwarp();
    } else if (warp < kDzWarp) {
        // ---------------------------------------------------------- epilogue
        // Per tile i:  A1(i) dx  ->  B(i-1) dz partial, dU flush, stage release  ->  A2(i) dw.
        const int ew = warp - 2;
        const int q = warp & 3;              // TMEM lane quarter == token rows 32q..32q+31
        const int h = ew >> 2;               // channel group of the slice (kCPW channels)
        const int row = 32 * q + lane;
        constexpr int CH = kCPW / 8;         // 16-byte chunks of the warp's channels in a row
        const uint32_t dxstage = sb + p.off_dx + (uint32_t)ew * kDxBuf;
        // staging rows of kCPW*2 bytes in the TMA store's 32- or 64-byte swizzle: the 16-byte
        // chunk index is XORed with address bits 7.. of the row start
        const uint32_t dxrow = (dxstage + lane * (2 * kCPW)) ^ ((((uint32_t)lane * (2 * kCPW) >> 7) & (CH - 1)) << 4);
        // dy rows r = row + k and x rows r = row + W-1-k of the 128-byte-swizzled tiles
        uint32_t dyr[W], xr[W];
#pragma unroll
        for (int k = 0; k < W; ++k) {
            uint32_t r = (uint32_t)(row + k);
            dyr[k] = (r * 128u) ^ ((r & 7u) << 4) ^ ((uint32_t)(CH * h) << 4);
            r = (uint32_t)(row + (W - 1) - k);
            xr[k] = (r * 128u) ^ ((r & 7u) << 4) ^ ((uint32_t)(CH * h) << 4);
        }
        // dw^T shared-memory tile: MN-major, 128B swizzle, atoms of 64 columns x 128 rows
        const uint32_t dwrow = sb + p.off_dw + (uint32_t)row * 128u;
        const uint32_t dwsw = (uint32_t)(row & 7) << 4;
        const uint32_t tl = tmem + ((uint32_t)(32 * q) << 16);

        struct Prev {
            int it, s, slice, b, t0, seg;
            bool last_of_slice;
        } pv = {-1, 0, 0, 0, 0, 0, false};
        // B: dz partial of a finished tile, its slice segment's dU partial, stage release
        auto phase_b = [&](const Prev &t) -> bool {
            if (!warp_wait(bar.mm2(), t.it & 1, abort, 256u, &g_fault_bwd)) return false;
            tc_fence_after();
            {
                // dz partial: every warp reads its group's share of the columns of its 32 rows
                const int tok = t.t0 + row;
                const int nc = p.R / Geo<G>::kGroups;
                float *dst = p.dz_part + ((size_t)t.slice * p.B * p.T + (size_t)t.b * p.T + tok) * p.R + h * nc;
                int c0 = 0;
#pragma unroll 1
                for (; c0 + 8 <= nc; c0 += 8) {
                    uint32_t v[8];
                    tmem_ld<8>(tl + p.tm_dz + h * nc + c0, v);
                    tmem_wait_ld_regs(v);
                    if (tok < p.T) {
                        *reinterpret_cast<uint4 *>(dst + c0) = make_uint4(v[0], v[1], v[2], v[3]);
                        *reinterpret_cast<uint4 *>(dst + c0 + 4) = make_uint4(v[4], v[5], v[6], v[7]);
                    }
                }
                if (c0 < nc) {   // nc = 4 (R = 16 with four channel groups)
                    uint32_t v[4];
                    tmem_ld<4>(tl + p.tm_dz + h * nc + c0, v);
                    tmem_wait_ld_regs(v);
                    if (tok < p.T) *reinterpret_cast<uint4 *>(dst + c0) = make_uint4(v[0], v[1], v[2], v[3]);
                }
            }
            if (t.last_of_slice && h < p.SCp / 128) {
                // lane j' of dU^T M-block h -> natural column g*W + k
                const int jp = 128 * h + row;
                const int jn = (jp % p.NGs) * W + jp / p.NGs;
                float *dst = p.du_part + ((size_t)t.slice * p.maxseg + t.seg) * p.R * p.SC + jn;
#pragma unroll 1
                for (int c0 = 0; c0 < p.R; c0 += 16) {
                    uint32_t v[16];
                    tmem_ld<16>(tl + p.tm_du + h * p.R + c0, v);     // all lanes: warp-collective
                    tmem_wait_ld_regs(v);
                    if (jp < p.SC) {
#pragma unroll
                        for (int m2 = 0; m2 < 16; ++m2) dst[(size_t)(c0 + m2) * p.SC] = __uint_as_float(v[m2]);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar.empty(t.s));
            return true;
        };

        int prev_slice = -1, seg = 0;
        bool ok = true;
        for (int i = tbeg; i < tend; ++i) {
            const int it = i - tbeg;
            const TileId id = tile_id(p, i);
            if (id.slice != prev_slice) {
                prev_slice = id.slice;
                seg = (int)blockIdx.x - owner_of((long long)id.slice * p.per_slice, p.n_tiles, gridDim.x);
            }
            const int s = it % p.stages, n = it / p.stages;
            if (!warp_wait(bar.full(s), n & 1, abort, 64u, &g_fault_bwd)) { ok = false; break; }
            const uint32_t st = sb + s * p.stage_bytes;
            const uint32_t dys = st, xs = st + p.xy_tile_bytes;
            // ---- A1: dx[t,c] = dy[t,c] + sum_k w[t+k,g,k] dy[t+k,c]
            // The warp's 16 channels are two 8-channel chunks, taken in batches of CB chunks:
            // a batch's shared-memory and TMEM loads are all issued before its first store
            // (the stores are ordered asm statements and would otherwise serialise the
            // loads); with many taps one chunk per batch keeps the registers in budget, and
            // the batch loop stays rolled so that the many-tap body fits the instruction cache.
            // A single batch's dy rows are loaded before the wait for the recomputed filters.
            constexpr int CB = (W * CH <= 8) ? CH : 1;
            constexpr int NGB = 8 * CB / G;                 // filter groups of a batch
            uint4 dpre[CB][W];
            if constexpr (CB == CH) {
#pragma unroll
                for (int cb = 0; cb < CB; ++cb)
#pragma unroll
                    for (int k = 0; k < W; ++k) dpre[cb][k] = lds128(dys + (dyr[k] ^ ((uint32_t)cb << 4)));
            }
            if (!warp_wait(bar.wfull(), it & 1, abort, 128u, &g_fault_bwd)) { ok = false; break; }
            tc_fence_after();
            if (lane == 0) bulk_wait_read<0>();
            __syncwarp();
#pragma unroll 1
            for (int c0 = 0; c0 < CH; c0 += CB) {
                uint4 du[CB][W];
#pragma unroll
                for (int cb = 0; cb < CB; ++cb)
#pragma unroll
                    for (int k = 0; k < W; ++k)
                        du[cb][k] = (CB == CH) ? dpre[cb][k] : lds128(dys + (dyr[k] ^ ((uint32_t)(c0 + cb) << 4)));
                uint32_t wr[W][NGB];
#pragma unroll
                for (int k = 0; k < W; ++k)
                    tmem_ld<NGB>(tl + p.tm_w + k * p.NGp + (kCPW * h + 8 * c0) / G, wr[k]);
                tmem_wait_ld();
#pragma unroll
                for (int k = 0; k < W; ++k)
#pragma unroll
                    for (int e = 0; e < NGB; ++e) asm volatile("" : "+r"(wr[k][e]));
                uint4 dxo[CB];
#pragma unroll
                for (int cb = 0; cb < CB; ++cb) {
                    const int gq = (8 * cb) / G;                   // chunk's first group within the batch
                    float dx[8];
                    if constexpr (G == 1) {
                        // channel pairs in packed fp32 FMAs (the same roundings as scalar fmaf)
                        uint64_t acc[4];
#pragma unroll
                        for (int k = 0; k < W; ++k) {
                            const uint32_t u[4] = {du[cb][k].x, du[cb][k].y, du[cb][k].z, du[cb][k].w};
#pragma unroll
                            for (int m = 0; m < 4; ++m) {
                                const uint64_t d2 = f2pack(bf16_lo(u[m]), bf16_hi(u[m]));
                                const uint64_t w2 = f2pack(__uint_as_float(wr[k][gq + 2 * m]),
                                                           __uint_as_float(wr[k][gq + 2 * m + 1]));
                                acc[m] = f2fma(w2, d2, k == 0 ? d2 : acc[m]);
                            }
                        }
#pragma unroll
                        for (int m = 0; m < 4; ++m) f2unpack(acc[m], dx[2 * m], dx[2 * m + 1]);
                    } else {
                        {
                            float d0[8];
                            unpack8(du[cb][0], d0);
#pragma unroll
                            for (int e = 0; e < 8; ++e) dx[e] = fmaf(__uint_as_float(wr[0][gq + e / G]), d0[e], d0[e]);
                        }
#pragma unroll
                        for (int k = 1; k < W; ++k) {
                            float dk[8];
                            unpack8(du[cb][k], dk);
#pragma unroll
                            for (int e = 0; e < 8; ++e) dx[e] = fmaf(__uint_as_float(wr[k][gq + e / G]), dk[e], dx[e]);
                        }
                    }
                    dxo[cb].x = pack_bf16x2(dx[0], dx[1]);
                    dxo[cb].y = pack_bf16x2(dx[2], dx[3]);
                    dxo[cb].z = pack_bf16x2(dx[4], dx[5]);
                    dxo[cb].w = pack_bf16x2(dx[6], dx[7]);
                }
#pragma unroll
                for (int cb = 0; cb < CB; ++cb) sts128(dxrow ^ ((uint32_t)(c0 + cb) << 4), dxo[cb]);
            }
            tc_fence_before();
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(bar.wempty());
                tma_store_3d(&tm_dx, dxstage, id.slice * kDt + kCPW * h, id.t0 + 32 * q, id.b);
                bulk_commit();
            }
            // ---- A2: dw[t,g,k] = sum_{c in g} dy[t,c] x[t-k,c], tap-major column k*NG + g,
            // in batches of CB chunks as A1.  A batch is computed into registers (pk) and
            // then stored; only the stores need the previous tile's dz / dU MMAs to be done
            // with the dw tile, so a single-batch A2 is computed before B waits for them.
            constexpr int NPK = (NG8 + 1) / 2;           // packed bf16 pairs per (chunk, tap)
            auto a2_compute = [&](int c0, uint32_t (&pk)[CB][W][NPK]) {
                uint4 d0[CB], xu[CB][W];
#pragma unroll
                for (int cb = 0; cb < CB; ++cb) {
                    d0[cb] = lds128(dys + (dyr[0] ^ ((uint32_t)(c0 + cb) << 4)));
#pragma unroll
                    for (int k = 0; k < W; ++k) xu[cb][k] = lds128(xs + (xr[k] ^ ((uint32_t)(c0 + cb) << 4)));
                }
#pragma unroll
                for (int cb = 0; cb < CB; ++cb)
#pragma unroll
                    for (int k = 0; k < W; ++k) {
                        if constexpr (G == 1) {
                            // one channel per group: dw = dy * x, exact in fp32 and rounded once
                            // to bf16, which is what the packed bf16 multiply computes
                            pk[cb][k][0] = bf16x2_mul(d0[cb].x, xu[cb][k].x);
                            pk[cb][k][1] = bf16x2_mul(d0[cb].y, xu[cb][k].y);
                            pk[cb][k][2] = bf16x2_mul(d0[cb].z, xu[cb][k].z);
                            pk[cb][k][3] = bf16x2_mul(d0[cb].w, xu[cb][k].w);
                        } else {
                            float dv[8], xv[8], dw[NG8];
                            unpack8(d0[cb], dv);
                            unpack8(xu[cb][k], xv);
#pragma unroll
                            for (int gl = 0; gl < NG8; ++gl) {
                                float acc = 0.f;
#pragma unroll
                                for (int e = gl * G; e < (gl + 1) * G; ++e) acc = fmaf(dv[e], xv[e], acc);
                                dw[gl] = acc;
                            }
#pragma unroll
                            for (int m2 = 0; m2 < NG8 / 2; ++m2) pk[cb][k][m2] = pack_bf16x2(dw[2 * m2], dw[2 * m2 + 1]);
                        }
                    }
            };
            auto a2_store = [&](int c0, const uint32_t (&pk)[CB][W][NPK]) {
#pragma unroll
                for (int cb = 0; cb < CB; ++cb) {
                    const int g8 = (kCPW * h + 8 * (c0 + cb)) / G;
#pragma unroll
                    for (int k = 0; k < W; ++k) {
                        const int jp = k * p.NGs + g8;                    // first tap-major column
                        const uint32_t atom = (uint32_t)(jp >> 6), within = (uint32_t)(jp & 63);
                        const uint32_t a = dwrow + atom * 16384u + ((((within >> 3) << 4) ^ dwsw) | ((within & 7) * 2));
                        if constexpr (NG8 == 8) {
                            sts128(a, make_uint4(pk[cb][k][0], pk[cb][k][1], pk[cb][k][2], pk[cb][k][3]));
                        } else if constexpr (NG8 == 4) {
                            sts64(a, pk[cb][k][0], pk[cb][k][1]);
                        } else {
                            sts32(a, pk[cb][k][0]);
                        }
                    }
                }
            };
            if constexpr (CB == CH) {
                uint32_t pk[CB][W][NPK];
                a2_compute(0, pk);
                // ---- B of the previous tile (its dz / dU MMAs ran during A1)
                if (pv.it >= 0 && !phase_b(pv)) { ok = false; break; }
                a2_store(0, pk);
            } else {
                // several batches (many taps): holding one across B cost more than it hid
                if (pv.it >= 0 && !phase_b(pv)) { ok = false; break; }
#pragma unroll 1
                for (int c0 = 0; c0 < CH; c0 += CB) {
                    uint32_t pk[CB][W][NPK];
                    a2_compute(c0, pk);
                    a2_store(c0, pk);
                }
            }
            tc_fence_before();
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar.dwready());
            pv.it = it;
            pv.s = s;
            pv.slice = id.slice;
            pv.b = id.b;
            pv.t0 = id.t0;
            pv.seg = seg;
            pv.last_of_slice = (i + 1 == tend) || ((i + 1) / p.per_slice != id.slice);
        }
        if (ok && pv.it >= 0) phase_b(pv);
        if (lane == 0) bulk_wait_all();
        __syncwarp();
    } else if (warp == kDzWarp) {
        // ---------------------------------------------------------- MMA issuer: dz partial
        // dz = dw Up^T once tile i's dw is written: A = dw tile (K-major view), B = Up slice
        // (K-major), 16 columns per step (+32 bytes within a 64-column atom, the next atom
        // every 4 steps).
        const uint64_t t_k128 = desc_tmpl(16, 1024, kSw128);
        const uint32_t i_dz = idesc_bf16(128, p.R, false, false);
        const int ksc = p.SC / 16;
        const uint32_t ubox = (uint32_t)(p.R * 128);
        const uint64_t st_wrap_a = (16384u - 96u) >> 4;   // next 64-column dw atom
        const uint64_t st_wrap_b = (ubox - 96u) >> 4;     // next 64-column Up box
        const uint32_t dw0 = sb + p.off_dw;
        int prev_slice = -1, v = -1, ub = 0;
        for (int i = tbeg; i < tend; ++i) {
            const int it = i - tbeg;
            const TileId id = tile_id(p, i);
            if (id.slice != prev_slice) {
                prev_slice = id.slice;
                ++v;
                ub = v % p.nU;
                if (!warp_wait(bar.uf(ub), (v / p.nU) & 1, abort, 4u, &g_fault_bwd)) break;
            }
            if (!warp_wait(bar.dwready(), it & 1, abort, 32u, &g_fault_bwd)) break;
            tc_fence_after();
            const uint32_t us = sb + p.off_u + ub * p.u_bytes;
            uint64_t da = desc_at(t_k128, dw0), db = desc_at(t_k128, us);
            for (int kk = 0; kk < ksc; ++kk) {
                if (elect_one()) mma_bf16_ss(tmem + p.tm_dz, da, db, i_dz, kk > 0 ? 1u : 0u);
                __syncwarp();
                const bool wrap = (kk & 3) == 3;
                da += wrap ? st_wrap_a : 2u;
                db += wrap ? st_wrap_b : 2u;
            }
            const bool last_of_slice = (i + 1 == tend) || ((i + 1) / p.per_slice != id.slice);
            if (elect_one()) {
                mma_commit(bar.mm2());
                if (last_of_slice) mma_commit(bar.ue(ub));
            }
            __syncwarp();
        }
        if (elect_one()) mma_commit(bar.done());
        __syncwarp();
    } else if (warp == kDuWarp) {
        // ---------------------------------------------------------- MMA issuer: dU partial
        // dU^T += dw^T z once tile i's dw is written: A = dw^T (MN-major), B = z tile rows
        // 0..127 (MN-major), 16 tokens per step; the accumulator restarts with each slice
        // segment of the CTA.
        const uint64_t t_dwt = desc_tmpl(16384, 1024, kSw128);
        const uint64_t t_zmn = desc_tmpl(128, p.z_slab, kSwNone);
        const uint32_t i_du = idesc_bf16(128, p.R, true, true);
        const int nmb = p.SCp / 128;
        const uint32_t dw0 = sb + p.off_dw;
        int prev_slice = -1;
        bool seg_first = true;
        for (int i = tbeg; i < tend; ++i) {
            const int it = i - tbeg;
            const TileId id = tile_id(p, i);
            if (id.slice != prev_slice) {
                prev_slice = id.slice;
                seg_first = true;
            }
            if (!warp_wait(bar.dwready(), it & 1, abort, 32u, &g_fault_bwd)) break;
            tc_fence_after();
            const uint32_t zs = sb + (it % p.stages) * p.stage_bytes + 2 * p.xy_tile_bytes;
            for (int mb = 0; mb < nmb; ++mb) {
                const uint32_t d = tmem + p.tm_du + mb * p.R;
                uint64_t da = desc_at(t_dwt, dw0 + mb * 32768u), db = desc_at(t_zmn, zs);
#pragma unroll
                for (int kk = 0; kk < kTt / 16; ++kk) {
                    if (elect_one()) mma_bf16_ss(d, da, db, i_du, (seg_first && kk == 0) ? 0u : 1u);
                    __syncwarp();
                    da += 2048u >> 4;
                    db += 256u >> 4;
                }
            }
            if (elect_one()) mma_commit(bar.mm2());
            __syncwarp();
            seg_first = false;
        }
        if (elect_one()) mma_commit(bar.done());
        __syncwarp();
    }

    __syncthreads();
    if (warp == 1) {
        if (lane == 0) mbar_wait(bar.done(), 0, abort, 0u, &g_fault_bwd);
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, p.tmem_cols);
    }
}

// Up[r, s*SC + k*NG + g] = U[r, s*SC + g*W + k]  (tap-major columns within each slice).
// Grid (ceil(N/2048), R): one row r per grid row; each thread writes 8 consecutive output
// columns with one 16-byte store (NG is a multiple of 8, so the 8 share one tap k and read
// source columns W apart).
__global__ void k_permute_u(const bf16 *__restrict__ U, bf16 *__restrict__ Up, int R, int N, int SC, int NG,
                            int W) {
    const int r = blockIdx.y;
    const int j = 8 * (blockIdx.x * blockDim.x + threadIdx.x);
    if (r >= R || j >= N) return;
    const int s = j / SC, jl = j - s * SC;
    const int k = jl / NG, g = jl - k * NG;
    const unsigned short *src = reinterpret_cast<const unsigned short *>(U) + (size_t)r * N + s * SC + g * W + k;
    uint32_t v[4];
#pragma unroll
    for (int m = 0; m < 4; ++m) v[m] = (uint32_t)src[(2 * m) * W] | ((uint32_t)src[(2 * m + 1) * W] << 16);
    *reinterpret_cast<uint4 *>(Up + (size_t)r * N + j) = make_uint4(v[0], v[1], v[2], v[3]);
}

// Both reductions in one launch (they are independent, so the small dU sum runs beside
// the dz sum instead of after it):
//   blocks [0, nb_dz):  dz[bt, :] = sum_s part_dz[s, bt, :]  (slices in order), grid-stride
//                       over float4 elements;
//   blocks [nb_dz, ..): dU[r, s*SC + j] = sum over the CTA segments of slice s of
//                       part_du[s, seg, r, j]  (in order); block nb_dz + r*nbx + bx covers row
//                       r, columns 4*(256*bx + thread) .. +3 (SC is a multiple of 8, so the
//                       four never straddle a slice).
__global__ void k_reduce(const float *__restrict__ part_dz, float *__restrict__ dz, int n_slices, size_t n4,
                         int nb_dz, const float *__restrict__ part_du, float *__restrict__ dU, int R, int SC,
                         int maxseg, int per_slice, int n_tiles, int grid, int nbx) {
    if ((int)blockIdx.x < nb_dz) {
        for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < n4; e += (size_t)nb_dz * blockDim.x) {
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int s = 0; s < n_slices; ++s) {
                const float4 v = reinterpret_cast<const float4 *>(part_dz)[(size_t)s * n4 + e];
                acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
            }
            reinterpret_cast<float4 *>(dz)[e] = acc;
        }
        return;
    }
    const int bid = (int)blockIdx.x - nb_dz;
    const int r = bid / nbx;
    const int N = SC * n_slices;
    const int j = 4 * ((bid - r * nbx) * (int)blockDim.x + (int)threadIdx.x);
    if (r >= R || j >= N) return;
    const int s = j / SC, jl = j - s * SC;
    const int nseg = owner_of((long long)(s + 1) * per_slice - 1, n_tiles, grid) -
                     owner_of((long long)s * per_slice, n_tiles, grid) + 1;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int seg = 0; seg < nseg; ++seg) {
        const float4 v = *reinterpret_cast<const float4 *>(part_du + (((size_t)s * maxseg + seg) * R + r) * SC + jl);
        acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
    }
    *reinterpret_cast<float4 *>(dU + (size_t)r * N + j) = acc;
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

bool plan_bwd(int B, int T, int D, int G, int W, int R, int grid, BwdParams &p) {
    if (!(R == 16 || R == 32 || R == 64)) return false;
    if (D % kDt || !(G == 1 || G == 2 || G == 4) || W < 1 || W > 8) return false;
    p.B = B; p.T = T; p.D = D; p.G = G; p.W = W; p.R = R;
    p.NGs = kDt / G;
    p.NGp = p.NGs < 16 ? 16 : p.NGs;
    p.SC = p.NGs * W;
    if (p.SC % 16) return false;
    p.SCp = (p.SC + 127) / 128 * 128;
    p.n_slices = D / kDt;
    p.tiles_per_seq = (T + kTt - 1) / kTt;
    p.per_slice = B * p.tiles_per_seq;
    const long long nt = (long long)p.n_slices * p.per_slice;
    if (nt >= (1ll << 31)) return false;
    p.n_tiles = (int)nt;
    if (grid > p.n_tiles) grid = p.n_tiles;
    int maxseg = 1;
    for (int s = 0; s < p.n_slices; ++s) {
        const int c0 = owner_of((long long)s * p.per_slice, p.n_tiles, grid);
        const int c1 = owner_of((long long)(s + 1) * p.per_slice - 1, p.n_tiles, grid);
        maxseg = std::max(maxseg, c1 - c0 + 1);
    }
    p.maxseg = maxseg;
    p.u_boxes = (p.SC + 63) / 64;
    // TMEM: w (W tap blocks) | dz | dU^T
    p.tm_w = 0;
    p.tm_dw = 0;   // unused: dw lives in shared memory only
    p.tm_dz = (uint32_t)(W * p.NGp + 31) / 32 * 32;
    p.tm_du = p.tm_dz + (uint32_t)R;
    const uint32_t used = p.tm_du + (uint32_t)(p.SCp / 128) * R;
    if (used > 512) return false;
    p.tmem_cols = 32;
    while (p.tmem_cols < used) p.tmem_cols *= 2;
    p.rows = kTt + W - 1;
    p.xy_tile_bytes = (p.rows * 128 + 1023) / 1024 * 1024;
    p.z_slab = (p.rows * 16 + 127) / 128 * 128;
    p.z_bytes = (uint32_t)(R / 8) * p.z_slab;
    p.stage_bytes = (2 * p.xy_tile_bytes + p.z_bytes + 1023) / 1024 * 1024;
    p.u_bytes = (uint32_t)(p.u_boxes * R * 128);
    const int options[4][2] = {{3, 2}, {3, 1}, {2, 2}, {2, 1}};   // (stages, U buffers)
    for (auto &o : options) {
        p.stages = o[0];
        p.nU = o[1];
        p.off_u = p.stages * p.stage_bytes;
        p.off_dw = p.off_u + p.nU * p.u_bytes;
        p.off_dw = (p.off_dw + 1023) / 1024 * 1024;
        p.off_dx = p.off_dw + (uint32_t)(p.SCp / 64) * 16384u;
        p.off_bar = p.off_dx + kDxStageBytes;
        if (p.off_bar + kBarBytes + 16 + 1024 <= kSmemLimit) return true;
    }
    return false;
}

template <int W, int G>
cudaError_t launch_t(const CUtensorMap *m, const BwdParams &p, int grid, cudaStream_t s) {
    auto kern = k_tc_lowrank_bwd<W, G>;
    const uint32_t smem = p.off_bar + kBarBytes + 16 + 1024;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, Geo<G>::kThreads, smem, s>>>(m[0], m[1], m[2], m[3], m[4], p);
    return cudaGetLastError();
}

template <int W>
cudaError_t launch_w(int G, const CUtensorMap *m, const BwdParams &p, int grid, cudaStream_t s) {
    switch (G) {
        case 1: return launch_t<W, 1>(m, p, grid, s);
        case 2: return launch_t<W, 2>(m, p, grid, s);
        default: return launch_t<W, 4>(m, p, grid, s);
    }
}

struct WsLayout {
    size_t up, dz, du, total;
};

WsLayout ws_layout(const BwdParams &p) {
    WsLayout l;
    const size_t N = (size_t)p.n_slices * p.SC;
    l.up = 0;
    l.dz = a256(l.up + (size_t)p.R * N * 2);
    l.du = a256(l.dz + (size_t)p.n_slices * p.B * p.T * p.R * 4);
    l.total = a256(l.du + (size_t)p.n_slices * p.maxseg * p.R * p.SC * 4);
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
                                  cudaStream_t s) {
    using namespace tcb;
    BwdParams p;
    const int grid = std::min(num_sms(), (D / kDt) * B * ((T + kTt - 1) / kTt));
    if (!plan_bwd(B, T, D, G, W, R, grid, p)) return cudaErrorNotSupported;
    const WsLayout l = ws_layout(p);
    uint8_t *w8 = (uint8_t *)ws;
    bf16 *Up = (bf16 *)(w8 + l.up);
    p.dz_part = (float *)(w8 + l.dz);
    p.du_part = (float *)(w8 + l.du);
    const int N = p.n_slices * p.SC;
    k_permute_u<<<dim3((N / 8 + 255) / 256, R), 256, 0, s>>>((const bf16 *)U, Up, R, N, p.SC, p.NGs, W);

    CUtensorMap m[5];
    const uint64_t dxyz[3] = {(uint64_t)D, (uint64_t)T, (uint64_t)B};
    const uint32_t bxy[3] = {(uint32_t)kDt, p.rows, 1};
    const uint64_t dzz[3] = {(uint64_t)R, (uint64_t)T, (uint64_t)B};
    const uint32_t bz[3] = {8, p.rows, 1};
    const uint64_t du[2] = {(uint64_t)N, (uint64_t)R};
    const uint32_t bu[2] = {64, (uint32_t)R};
    constexpr int kCPW = Geo<1>::kCPW;   // the same for every G
    static_assert(kCPW == 16 || kCPW == 32, "dx staging rows are 32 or 64 bytes");
    const uint32_t bdx[3] = {(uint32_t)kCPW, 32, 1};
    if (!make_map(&m[0], dy, 3, dxyz, bxy, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B) ||
        !make_map(&m[1], x, 3, dxyz, bxy, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B) ||
        !make_map(&m[2], z, 3, dzz, bz, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B) ||
        !make_map(&m[3], Up, 2, du, bu, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B) ||
        !make_map(&m[4], dx, 3, dxyz, bdx, kCPW == 16 ? CU_TENSOR_MAP_SWIZZLE_32B : CU_TENSOR_MAP_SWIZZLE_64B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_128B)) {
        set_last_error("dsc_bwd_lowrank: cuTensorMapEncodeTiled failed");
        return cudaErrorInvalidValue;
    }
    cudaError_t e;
    switch (W) {
        case 1: e = launch_w<1>(G, m, p, grid, s); break;
        case 2: e = launch_w<2>(G, m, p, grid, s); break;
        case 3: e = launch_w<3>(G, m, p, grid, s); break;
        case 4: e = launch_w<4>(G, m, p, grid, s); break;
        case 5: e = launch_w<5>(G, m, p, grid, s); break;
        case 6: e = launch_w<6>(G, m, p, grid, s); break;
        case 7: e = launch_w<7>(G, m, p, grid, s); break;
        default: e = launch_w<8>(G, m, p, grid, s); break;
    }
    if (e != cudaSuccess) return e;
    const size_t n4 = (size_t)B * T * R / 4;
    const int nb_dz = (int)std::min<size_t>((n4 + 255) / 256, 8192);
    const int nbx = (N / 4 + 255) / 256;
    k_reduce<<<nb_dz + nbx * R, 256, 0, s>>>(p.dz_part, dz, p.n_slices, n4, nb_dz, p.du_part, dU, R, p.SC,
                                             p.maxseg, p.per_slice, p.n_tiles, grid, nbx);
    return cudaGetLastError();
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
