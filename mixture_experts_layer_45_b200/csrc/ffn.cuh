// Step 3 of the layer: the grouped expert FFN (cookbook notebook "Mixture-
// of-experts and expert parallelism", section "Dispatch and gather": each
// expert is fc2(gelu(fc1(x))) on the tokens routed to it).
//
// Both GEMMs of an expert are C[M_e, N] = A[M_e, K] * W_e[N, K]^T with the
// operands K-contiguous: fc1 has A = xp (K = d), W = W1_e (N = ff) and the
// epilogue h = gelu(C + b1_e); fc2 has A = h (K = ff), W = W2_e (N = d) and
// the epilogue y = g_row * (C + b2_e).
//
// The expert row ranges live only on the device (offsets), so every CTA
// builds the same tile table from them and walks tiles t = blockIdx.x,
// blockIdx.x + gridDim.x, ... (persistent grid, no host synchronisation).
// Tile order: expert-major, then N tile, then M tile fastest, so CTAs that
// run together share the same weight panel through L2.
#pragma once

#include "common.cuh"

namespace moe {

enum FfnMode { kFc1Gelu = 0, kFc2Gate = 1 };

// SM clock of the grouped-FFN launches (moe_ffn_clock_enable / _read):
// while g_ffn_clock_on is set, thread 0 of every CTA records %clock64 and
// %globaltimer when it starts its tiles and when it is done (slots
// [mode][cta][0..3]), so that the host can divide cycles by nanoseconds:
// under the power cap the clock drops within a millisecond, faster than an
// outside sampler follows it.
constexpr int kClockCtas = 256;
__device__ int g_ffn_clock_on;
__device__ unsigned long long g_ffn_clock[2][kClockCtas][4];

__device__ __forceinline__ bool ffn_clock_on() { return *reinterpret_cast<volatile int*>(&g_ffn_clock_on) != 0; }

__device__ __forceinline__ void ffn_clock_mark(bool on, int mode, int slot) {
    if (on && threadIdx.x == 0 && blockIdx.x < kClockCtas) {
        unsigned long long c;
        asm volatile("mov.u64 %0, %%clock64;" : "=l"(c));
        g_ffn_clock[mode][blockIdx.x][slot] = c;
        g_ffn_clock[mode][blockIdx.x][slot + 1] = globaltimer_ns();
    }
}

// Shared always-on experts (notebook section "Exercises", item 3: every
// token also passes through a few experts outside the router) run as S
// extra row groups after the E routed ones, in the same launch: group E + s
// has `rows` rows (all tokens), reads A rows arow0 + s * astride ..., weight
// panel s of the shared weight tensor, and writes C rows crow0 + s * rows ...
// with gate 1.  S = 0 leaves only the routed groups.
struct SharedGroups {
    int S;
    int rows;
    int arow0, astride;
    int crow0;
};

constexpr int kMaxGroups = MOE_MAX_EXPERTS + MOE_MAX_SHARED;

struct TileTable {
    int start[kMaxGroups + 1];   // first tile of the group at each walk rank; start[G] = total
    int order[kMaxGroups];       // group at each walk rank
    int mtiles[kMaxGroups];      // M tiles of each group
    int arow[kMaxGroups];        // first A row of each group
    int crow[kMaxGroups];        // first C row (and row_gate / out_rows index)
    int rows[kMaxGroups];        // rows of each group
    int routed_tiles;            // tiles of the routed groups (ranks 0 .. E-1)
    int zip;                     // 0: plain walk; > 0: hot/cold interleave, positions per wave
};

// Must be called by all threads of the CTA; ends with __syncthreads().
// Routed group e < E covers rows offsets[e] .. offsets[e+1]-1 of A and C.
//
// zip > 0 (the number of CTAs, or CTA pairs, walking the tiles together)
// ranks the routed groups by M tiles, largest first (ties: lower index
// first), and decode_tile then interleaves the two ends of that list (see
// there).  zip = 0 keeps the groups in index order.  Shared groups always
// follow the routed ones.
__device__ __forceinline__ void build_tile_table(const int32_t* __restrict__ offsets, int E, const SharedGroups& sh,
                                                 int BM, int ntiles_n, TileTable& tt, int zip = 0) {
    pdl_wait();
    pdl_release();
    const int G = E + sh.S;
    for (int g = threadIdx.x; g < G; g += blockDim.x) {
        if (g < E) {
            const int lo = offsets[g];
            tt.arow[g] = lo;
            tt.crow[g] = lo;
            tt.rows[g] = offsets[g + 1] - lo;
        } else {
            const int s = g - E;
            tt.arow[g] = sh.arow0 + s * sh.astride;
            tt.crow[g] = sh.crow0 + s * sh.rows;
            tt.rows[g] = sh.rows;
        }
        tt.mtiles[g] = (tt.rows[g] + BM - 1) / BM;
    }
    __syncthreads();
    // walk rank of each group
    for (int g = threadIdx.x; g < G; g += blockDim.x) {
        int r = g;
        if (zip > 0 && g < E) {
            const int mg = tt.mtiles[g];
            r = 0;
            for (int h = 0; h < E; ++h) {
                const int mh = tt.mtiles[h];
                r += (mh > mg || (mh == mg && h < g)) ? 1 : 0;
            }
        }
        tt.order[r] = g;
    }
    __syncthreads();
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        constexpr int PER = (kMaxGroups + 31) / 32;
        int tl[PER];
        int sum = 0;
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const int r = lane * PER + i;
            tl[i] = (r < G) ? tt.mtiles[tt.order[r]] * ntiles_n : 0;
            sum += tl[i];
        }
        int incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        int run = incl - sum;
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const int r = lane * PER + i;
            if (r < G) tt.start[r] = run;
            run += tl[i];
        }
        if (lane == 31) tt.start[G] = incl;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        tt.routed_tiles = tt.start[E];
        tt.zip = zip;
    }
    __syncthreads();
}

struct TileCoord {
    int e, mt, nt;   // e: group (routed expert, or E + shared expert)
};

// Position t of the walk -> tile.
//
// With both routed and shared groups the walk interleaves them in
// proportion (position t is routed tile floor(t*Rt/N) when that count steps
// at t, else shared tile t - that count; a bijection since Rt <= N), so the
// CTAs running at any moment mix routed tiles, which stream their weight
// panels from HBM, with shared tiles, whose panels stay in L2 across their
// many M tiles.
//
// With tt.zip > 0 the routed positions alternate between the two ends of
// the size-ranked tile list: "front" positions take tiles 0, 1, 2, ... (the
// largest groups, whose weight panels serve many M tiles from L2), "back"
// positions take tiles Rt-1, Rt-2, ... (the smallest groups, each tile
// streaming its own panel from HBM).  So at any moment about half the CTAs
// compute from L2 while the others stream weights, instead of a phase of
// pure compute followed by a phase bound by HBM.  A position u of wave
// w = u / zip is a front one when u + w is even (zip even) or u is even
// (zip odd), so each CTA (position u mod zip) alternates between the two
// ends from wave to wave.  Front index = front positions before u; back
// index = the others; the two ranges meet in the middle: a bijection.
__device__ __forceinline__ TileCoord decode_tile(const TileTable& tt, int G, int t) {
    const int total = tt.start[G], rt = tt.routed_tiles;
    bool routed = true;
    if (rt > 0 && rt < total) {
        const int r0 = int((long long)t * rt / total);
        const int r1 = int((long long)(t + 1) * rt / total);
        routed = r1 > r0;
        t = routed ? r0 : rt + (t - r0);
    } else if (rt == 0) {
        routed = false;
    }
    if (routed && tt.zip > 0) {
        const int Z = tt.zip;
        const int u = t;
        int front_before;   // front positions in [0, u)
        bool front;
        if (Z & 1) {
            front = (u & 1) == 0;
            front_before = (u + 1) >> 1;
        } else {
            const int w = u / Z, c = u - w * Z;
            front = ((c + w) & 1) == 0;
            front_before = w * (Z >> 1) + ((w & 1) ? (c >> 1) : ((c + 1) >> 1));
        }
        t = front ? front_before : rt - 1 - (u - front_before);
    }
    int lo = 0, hi = G - 1;   // last rank r with start[r] <= t (groups with no tiles are skipped)
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (tt.start[mid] <= t) lo = mid; else hi = mid - 1;
    }
    // groups without tiles have start[r] == start[r+1], so the last rank with
    // start[r] <= t is the one whose range [start[r], start[r+1]) holds t
    TileCoord c;
    c.e = tt.order[lo];
    const int local = t - tt.start[lo];
    const int mt = tt.mtiles[c.e];
    c.nt = local / mt;
    c.mt = local - c.nt * mt;
    return c;
}

// ===========================================================================
// bf16 path: tcgen05.mma (kind::f16) with fp32 accumulators in tensor
// memory, operands brought to shared memory by TMA (128B swizzle).
//
// Warp roles (320 threads):
//   warp 0        TMA producer (one thread)
//   warp 1        tensor-memory allocator and MMA issuer (one thread)
//   warps 2..9    epilogue: warp w reads TMEM lane quarter w%4 and every
//                 other 32-column chunk (half (w-2)/4), adds the bias
//                 (staged once per tile in shared memory), applies GELU or
//                 the row gate, rounds to bf16 and stores rows masked to
//                 the expert's group
// Pipelines: STAGES shared-memory stages (full/empty mbarriers) and two
// accumulators of BN columns each (tfull/tempty mbarriers), so the
// epilogue of one tile overlaps the main loop of the next.
// ===========================================================================
constexpr int kTcBM = 128;
constexpr int kTcBK = 64;            // 64 bf16 = 128 B = one swizzle row
constexpr int kTcEpiWarps = 8;
constexpr int kTcThreads = 64 + 32 * kTcEpiWarps;
// threads of the single-CTA kernel with EPIW epilogue warps
constexpr int tc_threads(int epiw) { return 64 + 32 * epiw; }

// Per-warp shared-memory staging of the epilogue's output: the warp turns
// its lane-per-row values into row segments so that each global store
// instruction writes whole 32-byte sectors of a few rows instead of 16
// bytes of each of 32 rows.  kEpiSegB bytes (columns x 2) per row and
// round: 64 with up to eight epilogue warps, 32 with more (the staging of
// all epilogue warps then still fits beside the pipeline stages).
__host__ __device__ constexpr uint32_t epi_seg_bytes(int epiw) { return epiw <= 8 ? 64u : 32u; }
__host__ __device__ constexpr uint32_t epi_stage_bytes(int epiw) { return uint32_t(epiw) * 32u * epi_seg_bytes(epiw); }


template <int BN, int STAGES>
struct TcCfg {
    static constexpr uint32_t kABytes = kTcBM * kTcBK * 2;
    static constexpr uint32_t kBBytes = BN * kTcBK * 2;
    static constexpr uint32_t kStageBytes = kABytes + kBBytes;
    static constexpr uint32_t kTmemCols = (2 * BN <= 32) ? 32 : (2 * BN <= 64) ? 64 : (2 * BN <= 128) ? 128
                                         : (2 * BN <= 256) ? 256 : 512;
    // stages, then the epilogue warps' staging buffers (+ alignment slack)
    static constexpr size_t kSmemBytes = size_t(STAGES) * kStageBytes + 1024;
    static constexpr size_t smem_bytes(int epiw) { return kSmemBytes + epi_stage_bytes(epiw); }
};

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint4 v) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}
__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr)
                 : "memory");
    return v;
}

// TMA tile store (no multicast) of one staged box from shared memory, and
// the issuing thread's bulk-group bookkeeping
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, uint32_t src, int c0, int c1) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(src), "r"(c0), "r"(c1)
                 : "memory");
}
__device__ __forceinline__ void epi_bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// the staged box has been read out of shared memory
__device__ __forceinline__ void epi_bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// the stores are complete
__device__ __forceinline__ void epi_bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Two fp32 values in 64 bits (x in the low half) for sm_100's paired fp32
// instructions (add / mul / fma .rn.f32x2): each is the same IEEE operation
// on both halves, so a paired evaluation gives bit for bit what two scalar
// ones give, in half the instructions.
__device__ __forceinline__ uint64_t f2_pack(float x, float y) {
    return (uint64_t(__float_as_uint(y)) << 32) | __float_as_uint(x);
}
__device__ __forceinline__ float f2_x(uint64_t p) { return __uint_as_float(uint32_t(p)); }
__device__ __forceinline__ float f2_y(uint64_t p) { return __uint_as_float(uint32_t(p >> 32)); }
__device__ __forceinline__ uint64_t f2_splat(float v) { return f2_pack(v, v); }
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

// gelu_as (Abramowitz & Stegun eq. 7.1.26 erf) on two values at once: the
// same constants and the same operations in the same order, the FMA-pipe
// ones paired, the reciprocal and the exponential per value; bit for bit
// gelu_as of each half (1 - q is formed as fma(q, -1, 1), the same
// correctly rounded value).
__device__ __forceinline__ uint64_t gelu_as2(uint64_t v) {
    const uint64_t a = v & 0x7FFFFFFF7FFFFFFFull;                       // |v|
    const uint64_t d = fma2(f2_splat(0.2316418883f), a, f2_splat(1.0f));
    const uint64_t t = f2_pack(rcp_approx(f2_x(d)), rcp_approx(f2_y(d)));
    uint64_t poly = fma2(f2_splat(0.5307027145f), t, f2_splat(-0.7265760135f));
    poly = fma2(poly, t, f2_splat(0.7107068705f));
    poly = fma2(poly, t, f2_splat(-0.142248368f));
    poly = fma2(poly, t, f2_splat(0.127414796f));
    poly = mul2(poly, t);
    const uint64_t e2 = mul2(mul2(f2_splat(-0.72134752044448169f), v), v);
    const uint64_t q = mul2(poly, f2_pack(ex2_approx(f2_x(e2)), ex2_approx(f2_y(e2))));
    const uint64_t w = fma2(q, f2_splat(-1.0f), f2_splat(1.0f));         // 1 - q
    const uint64_t phi = f2_pack(f2_x(v) >= 0.f ? f2_x(w) : f2_x(q), f2_y(v) >= 0.f ? f2_y(w) : f2_y(q));
    return mul2(v, phi);
}

// moe_debug_gelu variant 2: the paired form, y[i] for i in pairs
__global__ void gelu2_probe_kernel(const float* __restrict__ x, float* __restrict__ y, int n) {
    for (int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x); i < n; i += 2 * gridDim.x * blockDim.x) {
        const float b = (i + 1 < n) ? x[i + 1] : 0.f;
        const uint64_t r = gelu_as2(f2_pack(x[i], b));
        y[i] = f2_x(r);
        if (i + 1 < n) y[i + 1] = f2_y(r);
    }
}

// One warp's share of a tile's epilogue.  The warp reads TMEM lane quarter
// q (accumulator rows q*32 .. q*32+31, one per lane) and the 32-column
// chunks sub, sub + EPIW/4, ... of the BN-column accumulator at `tacc`.  It
// loads its chunks in groups of at most two (64 registers), waits once per
// group, and calls release() (the warp's arrival on the accumulator's
// "empty" barrier) as soon as its last group is in registers, so the MMA
// can start the next-but-one tile while this one is still being written.
// Then bias (from global memory: the same 16 bytes for every lane, a
// broadcast), GELU (fc1) or the row gate (fc2) and bf16 rounding, row by
// row (lane = row) into the warp's staging buffer `stg` (32 rows x SEG
// bytes; 16-byte unit u of row r at unit u ^ swz(r): the layout of the
// TMA 64-byte / 32-byte swizzle, free of bank conflicts both row-wise and
// column-wise).  When all 32 rows are inside the group and C's rows are
// contiguous (`tma`), one lane stores the box with a TMA tile store
// through tmC (box {SEG / 2 columns, 32 rows}), so the output leaves
// through the copy engine rather than the load/store pipeline that the
// operand stream shares; otherwise each store instruction covers
// 32 / (SEG / 16) rows x SEG bytes, to row `crow` of C for rows inside the
// group (`valid`).  The warp's lane 0 waits for its boxes to be read out of
// the buffer before the buffer is rewritten; the caller waits for them to
// complete before the CTA exits.
template <int BN, int MODE, int EPIW, typename Release>
__device__ __forceinline__ void epilogue_tile_warp(uint32_t tacc, int q, int sub, int lane, bool valid, size_t crow,
                                                   int n0, int N, float g, const __nv_bfloat16* __restrict__ bb,
                                                   __nv_bfloat16* __restrict__ C, uint32_t stg, const CUtensorMap* tmC,
                                                   bool tma_rows, Release release) {
    constexpr int kSub = EPIW / 4;
    constexpr int kChunks = (BN / 32 + kSub - 1) / kSub;   // chunks per warp (the last may be past BN)
    constexpr int kGroup = kChunks < 2 ? kChunks : 2;
    constexpr int kSegB = int(epi_seg_bytes(EPIW));
    constexpr int kUnits = kSegB / 16;                     // 16-byte units per row and round
    constexpr int kRounds = 64 / kSegB;                    // rounds per 32-column chunk
    constexpr int kRowsPer = 32 / kUnits;                  // rows per store instruction
    static_assert(EPIW % 4 == 0 && EPIW >= 4, "whole lane quarters");
    // unit swizzle of row r: 4 units (64-byte rows) or 2 (32-byte rows)
    auto swz = [](int r) { return kUnits == 4 ? ((r >> 1) & 3) : ((r >> 2) & 1); };
    // the rows this lane stores (one per store instruction i) and their masks
    const unsigned vmask = __ballot_sync(0xffffffffu, valid);
    const bool tma = tma_rows && vmask == 0xffffffffu;   // warp-uniform
    size_t drow[kUnits];
#pragma unroll
    for (int i = 0; i < kUnits; ++i)
        drow[i] = size_t(__shfl_sync(0xffffffffu, static_cast<unsigned long long>(crow), i * kRowsPer + lane / kUnits));
    const int uu = lane % kUnits;
#pragma unroll
    for (int g0 = 0; g0 < kChunks; g0 += kGroup) {
        uint32_t r[kGroup][32];
#pragma unroll
        for (int j = 0; j < kGroup; ++j) {
            const int c = sub + (g0 + j) * kSub;
            if (g0 + j < kChunks && c < BN / 32)   // warp-uniform: the loads are warp-collective
                tmem_ld_32x32b_x32(tacc + (uint32_t(q * 32) << 16) + uint32_t(c * 32), r[j]);
        }
        tmem_ld_wait();
        if (g0 + kGroup >= kChunks) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) release();
        }
#pragma unroll
        for (int j = 0; j < kGroup; ++j) {
            const int c = sub + (g0 + j) * kSub;
            const int nb = n0 + c * 32;
            if (!(g0 + j < kChunks && c < BN / 32) || nb >= N) continue;   // warp-uniform
#pragma unroll
            for (int h = 0; h < kRounds; ++h) {
                if (lane == 0) epi_bulk_wait_read();   // the buffer's previous box is out
                __syncwarp();
                // this lane's row: kUnits units of 8 columns each
#pragma unroll
                for (int v = 0; v < kUnits; ++v) {
                    const int col = h * (kSegB / 2) + v * 8;   // within the chunk
                    uint4 u = make_uint4(0u, 0u, 0u, 0u);
                    if (nb + col < N) {
                        // bias[nb + col .. +8): one 16-byte load (N % 8 == 0, 16-byte aligned rows)
                        const uint4 bw = __ldg(reinterpret_cast<const uint4*>(bb + nb + col));
                        const uint32_t bwv[4] = {bw.x, bw.y, bw.z, bw.w};
                        uint32_t o[4];
#pragma unroll
                        for (int p = 0; p < 4; ++p) {
                            // columns col + 2p, col + 2p + 1 as one pair
                            const uint64_t acc = (uint64_t(r[j][col + 2 * p + 1]) << 32) | r[j][col + 2 * p];
                            const uint64_t cval = add2(acc, f2_pack(bf16_lo(bwv[p]), bf16_hi(bwv[p])));
                            const uint64_t y = (MODE == kFc1Gelu) ? gelu_as2(cval) : mul2(f2_splat(g), cval);
                            o[p] = pack_bf16x2(f2_x(y), f2_y(y));
                        }
                        u = make_uint4(o[0], o[1], o[2], o[3]);
                    }
                    st_shared_v4(stg + uint32_t(lane * kSegB + ((v ^ swz(lane)) << 4)), u);
                }
                if (tma) {
                    fence_proxy_async_smem();   // the TMA store (async proxy) reads these writes
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_2d(tmC, stg, nb + h * (kSegB / 2), int(drow[0]));
                        epi_bulk_commit();
                    }
                } else {
                    __syncwarp();
                    // row segments out: instruction i covers rows i*kRowsPer ..
#pragma unroll
                    for (int i = 0; i < kUnits; ++i) {
                        const int rr = i * kRowsPer + lane / kUnits;
                        const uint4 u = ld_shared_v4(stg + uint32_t(rr * kSegB + ((uu ^ swz(rr)) << 4)));
                        const int col = nb + h * (kSegB / 2) + uu * 8;
                        if (((vmask >> rr) & 1u) && col < N) *reinterpret_cast<uint4*>(C + drow[i] * N + col) = u;
                    }
                    __syncwarp();
                }
            }
        }
    }
}

// tmA2 / tmB2 / bias2: the shared experts' A rows and parameters (used when sh.S > 0).
// EPIW epilogue warps (a multiple of 4: EPIW / 4 warps share each TMEM lane
// quarter and split its 32-column chunks); fc1's GELU epilogue takes 16 so
// that it keeps up with the main loop at short K.
template <int BN, int STAGES, int MODE, int EPIW>
__global__ void __launch_bounds__(tc_threads(EPIW), 1)
ffn_tc_bf16_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const int32_t* __restrict__ offsets, int E, int N, int K,
                   const __nv_bfloat16* __restrict__ bias, const float* __restrict__ row_gate,
                   const int32_t* __restrict__ out_rows, __nv_bfloat16* __restrict__ C, SharedGroups sh,
                   const __grid_constant__ CUtensorMap tmA2, const __grid_constant__ CUtensorMap tmB2,
                   const __nv_bfloat16* __restrict__ bias2, int walk_zip, const __grid_constant__ CUtensorMap tmC,
                   int c_tma) {
    using Cfg = TcCfg<BN, STAGES>;
    static_assert(BN % 32 == 0 && BN >= 32 && BN <= 256, "BN: whole 32-column epilogue chunks, MMA N <= 256");
    __shared__ TileTable tt;
    __shared__ __align__(8) uint64_t full_bar[STAGES], empty_bar[STAGES];
    __shared__ __align__(8) uint64_t tfull_bar[2], tempty_bar[2], drain_bar;
    __shared__ uint32_t tmem_slot;
    __shared__ int abort_flag;
    extern __shared__ uint8_t dyn_smem[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dyn_smem) + 1023) & ~uintptr_t(1023));

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull_bar[a], 1);
            mbar_init(&tempty_bar[a], EPIW);   // one arrival per epilogue warp
        }
        mbar_init(&drain_bar, 1);
        abort_flag = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        if (sh.S > 0) {
            tma_prefetch_desc(&tmA2);
            tma_prefetch_desc(&tmB2);
        }
    }
    if (warp == 1) {
        tmem_alloc(&tmem_slot, Cfg::kTmemCols);
        tmem_relinquish();
        tc_fence_before();
    }
    const int ntn = (N + BN - 1) / BN;
    build_tile_table(offsets, E, sh, kTcBM, ntn, tt, walk_zip ? int(gridDim.x) : 0);   // ends with __syncthreads()
    tc_fence_after();
    const uint32_t tmem_base = tmem_slot;
    const int G = E + sh.S;
    const int total = tt.start[G];
    const int KB = (K + kTcBK - 1) / kTcBK;
    volatile int* abort_p = &abort_flag;
    const bool clock_on = ffn_clock_on();
    ffn_clock_mark(clock_on, MODE, 0);

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA producer ----------------
            int stage = 0;
            uint32_t phase = 0;
            int last_parity[STAGES];
            for (int s = 0; s < STAGES; ++s) last_parity[s] = -1;
            bool ok = true;
            for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
                const TileCoord tc = decode_tile(tt, G, t);
                const bool shared_g = tc.e >= E;
                const CUtensorMap* ma = shared_g ? &tmA2 : &tmA;
                const CUtensorMap* mb = shared_g ? &tmB2 : &tmB;
                const int widx = shared_g ? tc.e - E : tc.e;
                const int row0 = tt.arow[tc.e] + tc.mt * kTcBM;
                const int n0 = tc.nt * BN;
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait(&empty_bar[stage], phase ^ 1u, abort_p)) { ok = false; break; }
                    uint8_t* sa = smem + size_t(stage) * Cfg::kStageBytes;
                    uint8_t* sb = sa + Cfg::kABytes;
                    mbar_arrive_expect_tx(&full_bar[stage], Cfg::kStageBytes);
                    tma_load_2d(sa, ma, &full_bar[stage], kb * kTcBK, row0);
                    tma_load_3d(sb, mb, &full_bar[stage], kb * kTcBK, n0, widx);
                    last_parity[stage] = int(phase);
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
            }
            // every load this thread issued lands before the CTA exits
            // (immediate on the normal path, where the MMA consumed them)
            for (int s = 0; s < STAGES; ++s) {
                if (last_parity[s] < 0) continue;
                mbar_wait_drain(&full_bar[s], uint32_t(last_parity[s]));
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------- MMA issuer ----------------
            constexpr uint32_t idesc = idesc_bf16_f32(kTcBM, BN);
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
                if (!mbar_wait(&tempty_bar[acc], acc_phase ^ 1u, abort_p)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + uint32_t(acc * BN);
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait(&full_bar[stage], phase, abort_p)) { ok = false; break; }
                    tc_fence_after();
                    const uint8_t* sa = smem + size_t(stage) * Cfg::kStageBytes;
                    const uint64_t adesc = sdesc_kmajor_sw128(smem_u32(sa));
                    const uint64_t bdesc = sdesc_kmajor_sw128(smem_u32(sa + Cfg::kABytes));
#pragma unroll
                    for (int kk = 0; kk < kTcBK / 16; ++kk)
                        umma_f16(d_tmem, adesc + uint64_t(2 * kk), bdesc + uint64_t(2 * kk), idesc,
                                 (kb > 0 || kk > 0) ? 1u : 0u);
                    umma_commit(&empty_bar[stage]);
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                umma_commit(&tfull_bar[acc]);
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1u;
            }
            // every MMA this thread issued completes before TMEM is released
            umma_commit(&drain_bar);
            mbar_wait_drain(&drain_bar, 0);
        }
    } else {
        // ---------------- epilogue (warps 2 .. 1+EPIW) ----------------
        // Warp w takes TMEM lane quarter w % 4 and every (EPIW/4)-th
        // 32-column chunk from (w - 2) / 4 (epilogue_tile_warp).  Each warp
        // leaves the tile loop on its own when a wait gives up or the abort
        // flag is raised; no named barrier is involved.
        const int q = warp & 3;
        const int sub = (warp - 2) >> 2;
        const uint32_t stg = smem_u32(smem + size_t(STAGES) * Cfg::kStageBytes) +
                             uint32_t(warp - 2) * 32u * epi_seg_bytes(EPIW);
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int t = blockIdx.x; t < total; t += gridDim.x) {
            if (*abort_p) break;
            const TileCoord tc = decode_tile(tt, G, t);
            const bool shared_g = tc.e >= E;
            const int rows = tt.rows[tc.e];
            const int r_in = tc.mt * kTcBM + q * 32 + lane;
            const bool valid = r_in < rows;
            const size_t grow = size_t(tt.crow[tc.e]) + r_in;
            // destination row: the grouped row, or (direct output of a routed
            // group) the row out_rows names
            const size_t crow = (out_rows != nullptr && valid && !shared_g) ? size_t(out_rows[grow]) : grow;
            float g = 1.f;   // shared experts are ungated
            if (MODE == kFc2Gate && row_gate != nullptr && valid && !shared_g) g = row_gate[grow];
            const __nv_bfloat16* bb = shared_g ? bias2 + size_t(tc.e - E) * N : bias + size_t(tc.e) * N;
            // (uniform per warp: the TMEM loads are warp-collective)
            if (!__all_sync(0xffffffffu, mbar_wait(&tfull_bar[acc], acc_phase, abort_p))) break;
            tc_fence_after();
            uint64_t* tempty = &tempty_bar[acc];
            epilogue_tile_warp<BN, MODE, EPIW>(tmem_base + uint32_t(acc * BN), q, sub, lane, valid, crow, tc.nt * BN, N,
                                               g, bb, C, stg, &tmC, c_tma != 0,
                                               [tempty]() { mbar_arrive(tempty); });
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1u;
        }
        if (lane == 0) epi_bulk_wait_all();   // this warp's tile stores are complete
    }

    __syncthreads();
    ffn_clock_mark(clock_on, MODE, 2);
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, Cfg::kTmemCols);
    }
}

// ===========================================================================
// bf16 path on CTA pairs: tcgen05.mma.cta_group::2, 256 x 256 tiles.
//
// A cluster of two CTAs computes one 256-row x 256-column tile per step:
// CTA r loads A rows [m0 + 128r, +128) and weight rows [n0 + 128r, +128)
// (its halves of A and of the tile's N) into its own shared memory, both
// loads counting on CTA 0's `full` barrier; CTA 0's MMA thread issues the
// pair MMA and commits to both CTAs' `empty` / `tfull` barriers; each CTA's
// epilogue reads its 128 accumulator rows (all 256 columns) from its own
// tensor memory and signals CTA 0's `tempty` barrier.  Per CTA a k-block
// moves 32 KB for 128 x 256 x 64 MACs (the single-CTA tile moves 48 KB), so
// six stages fit in shared memory and the loads keep the tensor pipe fed
// at large K.  Same warp roles, tile table (M tiles of 256 rows), bounded
// waits and epilogue as ffn_tc_bf16_kernel.
// ===========================================================================
constexpr int kTc2BM = 256;          // rows per pair tile (128 per CTA)
constexpr int kTc2BN = 256;          // columns per pair tile (128 weight rows per CTA)

template <int STAGES>
struct Tc2Cfg {
    static constexpr uint32_t kABytes = 128 * kTcBK * 2;
    static constexpr uint32_t kBBytes = (kTc2BN / 2) * kTcBK * 2;
    static constexpr uint32_t kStageBytes = kABytes + kBBytes;
    static constexpr uint32_t kTmemCols = 2 * kTc2BN;   // two accumulators
    // stages, then the epilogue warps' staging buffers (+ alignment slack)
    static constexpr size_t kSmemBytes = size_t(STAGES) * kStageBytes + 1024;
    static constexpr size_t smem_bytes(int epiw) { return kSmemBytes + epi_stage_bytes(epiw); }
};

template <int STAGES, int MODE, int EPIW>
__global__ void __launch_bounds__(tc_threads(EPIW), 1)
ffn_tc2_bf16_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const int32_t* __restrict__ offsets, int E, int N, int K,
                    const __nv_bfloat16* __restrict__ bias, const float* __restrict__ row_gate,
                    const int32_t* __restrict__ out_rows, __nv_bfloat16* __restrict__ C, SharedGroups sh,
                    const __grid_constant__ CUtensorMap tmA2, const __grid_constant__ CUtensorMap tmB2,
                    const __nv_bfloat16* __restrict__ bias2, int walk_zip, const __grid_constant__ CUtensorMap tmC,
                    int c_tma) {
    using Cfg = Tc2Cfg<STAGES>;
    constexpr int BN = kTc2BN;
    __shared__ TileTable tt;
    __shared__ __align__(8) uint64_t full_bar[STAGES], empty_bar[STAGES];
    __shared__ __align__(8) uint64_t tfull_bar[2], tempty_bar[2], drain_bar;
    __shared__ uint32_t tmem_slot;
    __shared__ int abort_flag;
    extern __shared__ uint8_t dyn_smem[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dyn_smem) + 1023) & ~uintptr_t(1023));

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();   // 0: issues the pair MMAs
    const int pair = int(blockIdx.x >> 1), npairs = int(gridDim.x >> 1);
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full_bar[s], 1);    // CTA 0's copy counts both CTAs' loads
            mbar_init(&empty_bar[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull_bar[a], 1);
            mbar_init(&tempty_bar[a], 2 * EPIW);   // CTA 0's copy: every epilogue warp of the pair
        }
        mbar_init(&drain_bar, 1);
        abort_flag = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        if (sh.S > 0) {
            tma_prefetch_desc(&tmA2);
            tma_prefetch_desc(&tmB2);
        }
    }
    if (warp == 1) {
        tmem_alloc_pair(&tmem_slot, Cfg::kTmemCols);
        tmem_relinquish_pair();
        tc_fence_before();
    }
    const int ntn = (N + BN - 1) / BN;
    build_tile_table(offsets, E, sh, kTc2BM, ntn, tt, walk_zip ? npairs : 0);   // ends with __syncthreads()
    cluster_sync();   // both CTAs' barriers are initialised before any cross-CTA arrive
    tc_fence_after();
    const uint32_t tmem_base = tmem_slot;
    const int G = E + sh.S;
    const int total = tt.start[G];
    const int KB = (K + kTcBK - 1) / kTcBK;
    volatile int* abort_p = &abort_flag;
    const bool clock_on = ffn_clock_on();
    ffn_clock_mark(clock_on, MODE, 0);

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA producer (both CTAs) ----------------
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int t = pair; t < total && ok; t += npairs) {
                const TileCoord tc = decode_tile(tt, G, t);
                const bool shared_g = tc.e >= E;
                const CUtensorMap* ma = shared_g ? &tmA2 : &tmA;
                const CUtensorMap* mb = shared_g ? &tmB2 : &tmB;
                const int widx = shared_g ? tc.e - E : tc.e;
                const int row0 = tt.arow[tc.e] + tc.mt * kTc2BM + 128 * int(rank);
                const int n0 = tc.nt * BN + (BN / 2) * int(rank);
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait(&empty_bar[stage], phase ^ 1u, abort_p)) { ok = false; break; }
                    uint8_t* sa = smem + size_t(stage) * Cfg::kStageBytes;
                    uint8_t* sb = sa + Cfg::kABytes;
                    if (rank == 0) mbar_arrive_expect_tx(&full_bar[stage], 2 * Cfg::kStageBytes);
                    tma_load_2d_pair(sa, ma, &full_bar[stage], kb * kTcBK, row0);
                    tma_load_3d_pair(sb, mb, &full_bar[stage], kb * kTcBK, n0, widx);
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && rank == 0) {
            // ---------------- pair MMA issuer (CTA 0) ----------------
            constexpr uint32_t idesc = idesc_bf16_f32(kTc2BM, BN);
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            for (int t = pair; t < total && ok; t += npairs) {
                if (!mbar_wait(&tempty_bar[acc], acc_phase ^ 1u, abort_p)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + uint32_t(acc * BN);
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait(&full_bar[stage], phase, abort_p)) { ok = false; break; }
                    tc_fence_after();
                    const uint8_t* sa = smem + size_t(stage) * Cfg::kStageBytes;
                    const uint64_t adesc = sdesc_kmajor_sw128(smem_u32(sa));
                    const uint64_t bdesc = sdesc_kmajor_sw128(smem_u32(sa + Cfg::kABytes));
#pragma unroll
                    for (int kk = 0; kk < kTcBK / 16; ++kk)
                        umma_f16_pair(d_tmem, adesc + uint64_t(2 * kk), bdesc + uint64_t(2 * kk), idesc,
                                      (kb > 0 || kk > 0) ? 1u : 0u);
                    umma_commit_pair(&empty_bar[stage], 0x3);
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                umma_commit_pair(&tfull_bar[acc], 0x3);
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1u;
            }
            // every pair MMA completes (in both CTAs' view) before teardown
            umma_commit_pair(&drain_bar, 0x3);
        }
    } else {
        // ---------------- epilogue (warps 2 .. 1+EPIW of each CTA) ----------------
        // As in ffn_tc_bf16_kernel: each CTA's warps read their own 128
        // accumulator rows (the tile's rows 128*rank ..); every warp of the
        // pair arrives on CTA 0's "empty" barrier (CTA 1 through mapa).
        const int q = warp & 3;
        const int sub = (warp - 2) >> 2;
        const uint32_t stg = smem_u32(smem + size_t(STAGES) * Cfg::kStageBytes) +
                             uint32_t(warp - 2) * 32u * epi_seg_bytes(EPIW);
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int t = pair; t < total; t += npairs) {
            if (*abort_p) break;
            const TileCoord tc = decode_tile(tt, G, t);
            const bool shared_g = tc.e >= E;
            const int rows = tt.rows[tc.e];
            const int r_in = tc.mt * kTc2BM + 128 * int(rank) + q * 32 + lane;
            const bool valid = r_in < rows;
            const size_t grow = size_t(tt.crow[tc.e]) + r_in;
            const size_t crow = (out_rows != nullptr && valid && !shared_g) ? size_t(out_rows[grow]) : grow;
            float g = 1.f;
            if (MODE == kFc2Gate && row_gate != nullptr && valid && !shared_g) g = row_gate[grow];
            const __nv_bfloat16* bb = shared_g ? bias2 + size_t(tc.e - E) * N : bias + size_t(tc.e) * N;
            // (uniform per warp: the TMEM loads are warp-collective)
            if (!__all_sync(0xffffffffu, mbar_wait(&tfull_bar[acc], acc_phase, abort_p))) break;
            tc_fence_after();
            uint64_t* tempty = &tempty_bar[acc];
            epilogue_tile_warp<BN, MODE, EPIW>(tmem_base + uint32_t(acc * BN), q, sub, lane, valid, crow, tc.nt * BN, N,
                                               g, bb, C, stg, &tmC, c_tma != 0,
                                               [tempty, rank]() {
                                                   if (rank == 0) mbar_arrive(tempty);
                                                   else mbar_arrive_remote(tempty, 0);
                                               });
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1u;
        }
        if (lane == 0) epi_bulk_wait_all();   // this warp's tile stores are complete
    }

    // teardown: every pair MMA has completed (it reads both CTAs' shared
    // memory and writes both tensor memories) before either CTA frees
    // anything or exits
    if (warp == 1 && lane == 0) {
        mbar_wait_drain(&drain_bar, 0);
    }
    __syncthreads();
    cluster_sync();
    ffn_clock_mark(clock_on, MODE, 2);
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, Cfg::kTmemCols);
    }
}

}  // namespace moe
