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
// Warp roles (persistent CTAs, one per SM, each owning a contiguous range of tiles in
// slice-major order so that the U slice changes rarely):
//   warp 0  TMA producer (x, z per tile; U per slice), 4-stage ring
//   warp 1  TMEM allocator and MMA issuer (one thread), double-buffered accumulator
//   warps 2-9  epilogue: warp w reads TMEM lanes 32*(w%4).. (its 32 tokens) and handles
//              32 channels (half the slice); one token row per thread.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstdio>
#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"

namespace dsc {
namespace tc {

__device__ unsigned int g_fault = 0;

constexpr int kTt = 128;          // tokens per tile (MMA M)
constexpr int kDt = 64;           // channels per slice
constexpr int kEpiWarps = 8;
constexpr int kThreads = 32 * (2 + kEpiWarps);
constexpr int kYBuf = 32 * 64;    // one warp's y staging: 32 rows x 32 bf16 channels

struct FwdParams {
    int B, T, D, G, R;
    int per_slice;            // B * tiles_per_seq
    int tiles_per_seq;
    int n_tiles;
    int slice_cols;           // (64/G)*W
    int n_pad;                // slice_cols rounded up to 16
    int u_boxes;              // ceil(n_pad / 64) TMA boxes of 64 columns
    int bufcols, nbuf, tmem_cols;
    int stages, nU;
    uint32_t x_stage_tx, x_stage_bytes, z_stage_bytes, u_bytes;
    uint32_t off_x, off_z, off_u, off_y, off_bar;
    uint32_t z_layout;        // swizzle of the z tile (32/64/128-byte rows)
};

// Barrier slots in shared memory (in units of 8 bytes) for a ring of `S` stages.
struct Bars {
    uint32_t base;
    int S;
    __device__ uint32_t full(int s) const { return base + 8 * s; }
    __device__ uint32_t empty(int s) const { return base + 8 * (4 + s); }
    __device__ uint32_t accf(int a) const { return base + 8 * (8 + a); }
    __device__ uint32_t acce(int a) const { return base + 8 * (10 + a); }
    __device__ uint32_t uf(int u) const { return base + 8 * (12 + u); }
    __device__ uint32_t ue(int u) const { return base + 8 * (14 + u); }
    __device__ uint32_t done() const { return base + 8 * 16; }
};
constexpr uint32_t kBarBytes = 8 * 17;

__device__ __forceinline__ void unpack8(const uint4 &u, float (&v)[8]) {
    v[0] = bf16_lo(u.x); v[1] = bf16_hi(u.x);
    v[2] = bf16_lo(u.y); v[3] = bf16_hi(u.y);
    v[4] = bf16_lo(u.z); v[5] = bf16_hi(u.z);
    v[6] = bf16_lo(u.w); v[7] = bf16_hi(u.w);
}

// Columns of the chunk's filter taps, read from TMEM into wr[]:
//   GC <= 8: 8/GC groups x W taps, group-major (column gl*W + k), loaded as W pieces of
//            8/GC columns, each piece aligned to its width;
//   GC == 16 (any G >= 16): one group, W columns, loaded one by one.
template <int W, int GC>
struct Taps {
    static constexpr int PIECE = GC <= 8 ? 8 / GC : 1;
    static constexpr int NCOL = PIECE * W;
};

template <int W, int GC>
__global__ void __launch_bounds__(kThreads, 1)
k_tc_lowrank_fwd(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_z,
                 const __grid_constant__ CUtensorMap tm_u, const __grid_constant__ CUtensorMap tm_y,
                 const FwdParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const uint32_t sb = smem_u32(smem);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const Bars bar{sb + p.off_bar, p.stages};
    uint32_t *tmem_holder = (uint32_t *)(smem + p.off_bar + kBarBytes);
    volatile int *abort = (volatile int *)(smem + p.off_bar + kBarBytes + 8);

    if (threadIdx.x == 0) {
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(bar.full(s), 1);
            mbar_init(bar.empty(s), kEpiWarps);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(bar.accf(a), 1);
            mbar_init(bar.acce(a), kEpiWarps);
            mbar_init(bar.uf(a), 1);
            mbar_init(bar.ue(a), 1);
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
    const int S = p.stages;

    if (warp == 0) {
        // ---------------------------------------------------------- TMA producer
        if (lane == 0) {
            int prev = -1, v = -1;
            for (int i = tbeg; i < tend; ++i) {
                const int it = i - tbeg;
                const int slice = i / p.per_slice, rem = i % p.per_slice;
                const int b = rem / p.tiles_per_seq, t0 = (rem % p.tiles_per_seq) * kTt;
                if (slice != prev) {
                    prev = slice;
                    ++v;
                    const int ub = v % p.nU, un = v / p.nU;
                    if (!mbar_wait(bar.ue(ub), (un & 1) ^ 1, abort, 1u, &g_fault)) break;
                    mbar_arrive_expect_tx(bar.uf(ub), p.u_bytes);
                    const uint32_t ud = sb + p.off_u + ub * p.u_bytes;
                    for (int bx = 0; bx < p.u_boxes; ++bx)
                        tma_load_2d(ud + bx * (uint32_t)(p.R * 128), &tm_u, bar.uf(ub),
                                    slice * p.slice_cols + 64 * bx, 0);
                }
                const int s = it % S, n = it / S;
                if (!mbar_wait(bar.empty(s), (n & 1) ^ 1, abort, 2u, &g_fault)) break;
                mbar_arrive_expect_tx(bar.full(s), p.x_stage_tx + p.z_stage_bytes);
                tma_load_3d(sb + p.off_x + s * p.x_stage_bytes, &tm_x, bar.full(s), slice * kDt,
                            t0 - (W - 1), b);
                tma_load_3d(sb + p.off_z + s * p.z_stage_bytes, &tm_z, bar.full(s), 0, t0, b);
            }
            // Let every load this warp issued land before the CTA can exit.
            const int issued = tend - tbeg;
            for (int s = 0; s < S && s < issued; ++s) {
                const int last = issued - 1 - ((issued - 1 - s) % S);   // last tile using stage s
                mbar_wait(bar.full(s), (last / S) & 1, abort, 0u, &g_fault);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const int nchunks = (p.n_pad + 255) / 256;
            const uint32_t zsbo = 8u * p.R * 2u;
            int prev = -1, v = -1, ub = 0;
            for (int i = tbeg; i < tend; ++i) {
                const int it = i - tbeg;
                const int slice = i / p.per_slice;
                if (slice != prev) {
                    prev = slice;
                    ++v;
                    ub = v % p.nU;
                    if (!mbar_wait(bar.uf(ub), (v / p.nU) & 1, abort, 4u, &g_fault)) break;
                }
                const int s = it % S, n = it / S;
                const int a = it % p.nbuf, m = it / p.nbuf;
                if (!mbar_wait(bar.full(s), n & 1, abort, 8u, &g_fault)) break;
                if (!mbar_wait(bar.acce(a), (m & 1) ^ 1, abort, 16u, &g_fault)) break;
                tc_fence_after();
                const uint32_t d = tmem + a * p.bufcols;
                const uint32_t za = sb + p.off_z + s * p.z_stage_bytes;
                const uint32_t ua = sb + p.off_u + ub * p.u_bytes;
                for (int nc = 0; nc < nchunks; ++nc) {
                    const int ncols = min(256, p.n_pad - 256 * nc);
                    const uint32_t idesc = idesc_bf16(128, ncols, false, true);
                    for (int kk = 0; kk < p.R / 16; ++kk) {
                        const uint64_t ad = smem_desc(za + kk * 32, 16, zsbo, p.z_layout);
                        const uint64_t bd = smem_desc(ua + nc * 4 * (uint32_t)(p.R * 128) + kk * 2048,
                                                      (uint32_t)(p.R * 128), 1024, kSw128);
                        mma_bf16_ss(d + 256 * nc, ad, bd, idesc, kk > 0 ? 1u : 0u);
                    }
                }
                mma_commit(bar.accf(a));
                const bool last_of_slice = (i + 1 == tend) || ((i + 1) / p.per_slice != slice);
                if (last_of_slice) mma_commit(bar.ue(ub));
            }
            mma_commit(bar.done());
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------- epilogue
        using TP = Taps<W, GC>;
        const int q = warp & 3;              // TMEM lane quarter == token rows 32q..32q+31
        const int h = (warp - 2) >> 2;       // channel half of the slice
        const int row = 32 * q + lane;       // token row in the tile
        const uint32_t ybase = sb + p.off_y + (uint32_t)(warp - 2) * 2 * kYBuf;
        uint8_t *ygen = smem + p.off_y + (warp - 2) * 2 * kYBuf;
        int yc = 0;
        for (int i = tbeg; i < tend; ++i) {
            const int it = i - tbeg;
            const int slice = i / p.per_slice, rem = i % p.per_slice;
            const int b = rem / p.tiles_per_seq, t0 = (rem % p.tiles_per_seq) * kTt;
            const int s = it % S, n = it / S;
            const int a = it % p.nbuf, m = it / p.nbuf;
            if (!mbar_wait(bar.full(s), n & 1, abort, 32u, &g_fault)) break;
            if (!mbar_wait(bar.accf(a), m & 1, abort, 64u, &g_fault)) break;
            tc_fence_after();
            const int yb = yc & 1;
            if (lane == 0) bulk_wait_read<1>();
            __syncwarp();
            const uint8_t *xs = smem + p.off_x + s * p.x_stage_bytes;
            const uint32_t tl = tmem + ((uint32_t)(32 * q) << 16) + a * p.bufcols;
#pragma unroll
            for (int cq = 0; cq < 4; ++cq) {
                const int c8 = 32 * h + 8 * cq;          // first channel of the chunk in the slice
                uint32_t wr[TP::NCOL];
                if (GC <= 8) {
                    const uint32_t col = (uint32_t)((c8 / GC) * W);
#pragma unroll
                    for (int m2 = 0; m2 < W; ++m2) tmem_ld<TP::PIECE>(tl + col + m2 * TP::PIECE, &wr[m2 * TP::PIECE]);
                } else {
                    const uint32_t col = (uint32_t)((c8 / p.G) * W);
#pragma unroll
                    for (int k = 0; k < W; ++k) tmem_ld<1>(tl + col + k, &wr[k]);
                }
                float xv[W][8];
#pragma unroll
                for (int k = 0; k < W; ++k) {
                    const int rw = row + (W - 1) - k;
                    const int ch = (4 * h + cq) ^ (rw & 7);
                    const uint4 u = *reinterpret_cast<const uint4 *>(xs + rw * 128 + ch * 16);
                    unpack8(u, xv[k]);
                }
                tmem_wait_ld_regs(wr);
                float out[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int gl = GC <= 8 ? e / GC : 0;
                    float acc = xv[0][e];
#pragma unroll
                    for (int k = 0; k < W; ++k) acc = fmaf(__uint_as_float(wr[gl * W + k]), xv[k][e], acc);
                    out[e] = acc;
                }
                uint4 o;
                o.x = pack_bf16x2(out[0], out[1]);
                o.y = pack_bf16x2(out[2], out[3]);
                o.z = pack_bf16x2(out[4], out[5]);
                o.w = pack_bf16x2(out[6], out[7]);
                const int pc = cq ^ ((lane >> 1) & 3);   // 64-byte swizzle of the staging rows
                *reinterpret_cast<uint4 *>(ygen + yb * kYBuf + lane * 64 + pc * 16) = o;
            }
            tc_fence_before();
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(bar.acce(a));
                mbar_arrive(bar.empty(s));
                tma_store_3d(&tm_y, ybase + yb * kYBuf, slice * kDt + 32 * h, t0 + 32 * q, b);
                bulk_commit();
            }
            ++yc;
        }
        if (lane == 0) bulk_wait_all();
        __syncwarp();
    }

    __syncthreads();
    if (warp == 1) {
        if (lane == 0) mbar_wait(bar.done(), 0, abort, 0u, &g_fault);
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, p.tmem_cols);
    }
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
              CUtensorMapSwizzle sw) {
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
                           bdim, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
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

bool plan_fwd(int B, int T, int D, int G, int W, int R, FwdParams &p) {
    if (!(R == 16 || R == 32 || R == 64)) return false;
    if (D % kDt || !is_pow2(G) || G > 64 || W < 1 || W > 8) return false;
    p.B = B; p.T = T; p.D = D; p.G = G; p.R = R;
    p.slice_cols = (kDt / G) * W;
    if (p.slice_cols % 8) return false;           // U slice start must be 16-byte aligned for TMA
    p.n_pad = (p.slice_cols + 15) / 16 * 16;
    p.u_boxes = (p.n_pad + 63) / 64;
    p.tiles_per_seq = (T + kTt - 1) / kTt;
    p.per_slice = B * p.tiles_per_seq;
    const long long nt = (long long)(D / kDt) * p.per_slice;
    if (nt >= (1ll << 31)) return false;
    p.n_tiles = (int)nt;
    p.bufcols = p.n_pad;
    p.nbuf = (2 * p.n_pad <= 512) ? 2 : 1;
    int cols = 32;
    while (cols < p.nbuf * p.bufcols) cols *= 2;
    p.tmem_cols = cols;
    p.x_stage_tx = (uint32_t)(kDt * 2 * (kTt + W - 1));
    p.x_stage_bytes = (p.x_stage_tx + 1023) / 1024 * 1024;
    p.z_stage_bytes = (uint32_t)(kTt * R * 2);
    p.u_bytes = (uint32_t)(p.u_boxes * R * 128);
    p.z_layout = R == 16 ? kSw32 : (R == 32 ? kSw64 : kSw128);
    const int options[5][2] = {{4, 2}, {3, 2}, {4, 1}, {3, 1}, {2, 1}};
    for (auto &o : options) {
        const uint32_t off_x = 0;
        const uint32_t off_z = off_x + o[0] * p.x_stage_bytes;
        const uint32_t off_u = off_z + o[0] * p.z_stage_bytes;
        const uint32_t off_y = off_u + o[1] * p.u_bytes;
        const uint32_t off_bar = off_y + kEpiWarps * 2 * kYBuf;
        const uint32_t total = off_bar + kBarBytes + 16 + 1024;
        if (total <= kSmemLimit) {
            p.stages = o[0];
            p.nU = o[1];
            p.off_x = off_x; p.off_z = off_z; p.off_u = off_u; p.off_y = off_y; p.off_bar = off_bar;
            return true;
        }
    }
    return false;
}

uint32_t smem_bytes(const FwdParams &p) { return p.off_bar + kBarBytes + 16 + 1024; }

template <int W, int GC>
cudaError_t launch_fwd_t(const CUtensorMap &mx, const CUtensorMap &mz, const CUtensorMap &mu,
                         const CUtensorMap &my, const FwdParams &p, cudaStream_t s) {
    auto kern = k_tc_lowrank_fwd<W, GC>;
    const uint32_t smem = smem_bytes(p);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int grid = std::min(p.n_tiles, num_sms());
    kern<<<grid, kThreads, smem, s>>>(mx, mz, mu, my, p);
    return cudaGetLastError();
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
                                  int D, int G, int W, int R, cudaStream_t s) {
    using namespace tc;
    FwdParams p;
    if (!plan_fwd(B, T, D, G, W, R, p)) return cudaErrorNotSupported;
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
    if (!make_map(&mx, x, 3, dx, bx, CU_TENSOR_MAP_SWIZZLE_128B) || !make_map(&mz, z, 3, dz, bz, zsw) ||
        !make_map(&mu, U, 2, du, bu, CU_TENSOR_MAP_SWIZZLE_128B) ||
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

bool tc_lowrank_bwd_supported(int, int, int, int, int, int, bool) { return false; }

size_t tc_lowrank_bwd_workspace(int, int, int, int, int, int) { return 0; }

cudaError_t launch_tc_lowrank_bwd(const void *, const void *, const void *, const void *, void *, float *,
                                  float *, void *, int, int, int, int, int, int, cudaStream_t) {
    return cudaErrorNotSupported;
}

unsigned read_device_fault(bool reset) {
    unsigned v = 0;
    if (cudaMemcpyFromSymbol(&v, tc::g_fault, sizeof(v)) != cudaSuccess) return 0xffffffffu;
    if (reset) {
        const unsigned z = 0;
        cudaMemcpyToSymbol(tc::g_fault, &z, sizeof(z));
    }
    return v;
}

}  // namespace dsc
