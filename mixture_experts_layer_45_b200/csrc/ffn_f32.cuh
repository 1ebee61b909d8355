// Step 3 of the layer for fp32 layers: the grouped expert FFN (cookbook
// notebook "Mixture-of-experts and expert parallelism", section "Dispatch
// and gather") on the tensor cores by three-pass TF32.  The tile table, the
// tile walk and the TMEM/TMA primitives are those of ffn.cuh.
#pragma once

#include "ffn.cuh"

namespace moe {

// ===========================================================================
// fp32 path: three-pass TF32 on the tensor cores (error-compensated).
//
// Each fp32 operand v is split into hi = v rounded to TF32 (low 13 mantissa
// bits cleared, round to nearest) and lo = v - hi (exact in fp32, |lo| <=
// 2^-11 |hi|); then A B^T = hi_A hi_B^T + hi_A lo_B^T + lo_A hi_B^T + lo_A lo_B^T
// and the last product, about 2^-22 of the result, is dropped.  Each kept
// product is a tcgen05.mma kind::tf32 with fp32 accumulation in tensor
// memory, so the result carries fp32-level error (the split-precision
// scheme of Ootomo & Yokota 2022) at the tensor cores' TF32 rate.
//
// Warp roles (576 threads):
//   warp 0        TMA producer: raw fp32 A and W tiles, 32 columns (128 B)
//                 of K per stage, 128B swizzle
//   warp 1        TMEM allocator and MMA issuer: 3 MMAs per K step of 8
//   warps 2..9    epilogue, as the bf16 kernel, fp32 stores
//   warps 10..17  converters: for each landed stage, hi in place and lo
//                 into the stage's lo tiles (same swizzled positions), then a
//                 proxy fence so the tensor cores see the generic writes
// ===========================================================================
constexpr int kTfBK = 32;            // 32 fp32 = 128 B = one swizzle row
constexpr int kTfConvWarps = 8;
constexpr int kTfThreads = 64 + 32 * kTcEpiWarps + 32 * kTfConvWarps;

template <int BN, int STAGES>
struct TfCfg {
    static constexpr uint32_t kABytes = kTcBM * kTfBK * 4;
    static constexpr uint32_t kBBytes = BN * kTfBK * 4;
    static constexpr uint32_t kLoadBytes = kABytes + kBBytes;        // what TMA brings per stage
    static constexpr uint32_t kStageBytes = 2 * kLoadBytes;          // + the lo tiles
    static constexpr uint32_t kTmemCols = (2 * BN <= 256) ? 256 : 512;
    static constexpr size_t kSmemBytes = size_t(STAGES) * kStageBytes + 1024;
};

__device__ __forceinline__ float tf32_round(float v) {
    // round to nearest on bit 13 (ties away from zero); inf / nan pass through
    const uint32_t u = __float_as_uint(v);
    if ((u & 0x7F800000u) == 0x7F800000u) return v;
    return __uint_as_float((u + 0x1000u) & 0xFFFFE000u);
}

template <int BN, int STAGES, int MODE>
__global__ void __launch_bounds__(kTfThreads, 1)
ffn_tc_f32x3_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const int32_t* __restrict__ offsets, int E, int N, int K,
                    const float* __restrict__ bias, const float* __restrict__ row_gate,
                    const int32_t* __restrict__ out_rows, float* __restrict__ C, SharedGroups sh,
                    const __grid_constant__ CUtensorMap tmA2, const __grid_constant__ CUtensorMap tmB2,
                    const float* __restrict__ bias2, int walk_zip) {
    using Cfg = TfCfg<BN, STAGES>;
    static_assert(BN % 32 == 0 && BN >= 32 && BN <= 256, "BN: whole 32-column epilogue chunks, MMA N <= 256");
    __shared__ TileTable tt;
    __shared__ __align__(8) uint64_t full_bar[STAGES], conv_bar[STAGES], empty_bar[STAGES];
    __shared__ __align__(8) uint64_t tfull_bar[2], tempty_bar[2], drain_bar;
    __shared__ uint32_t tmem_slot;
    __shared__ int abort_flag;
    __shared__ float sbias[BN];
    extern __shared__ uint8_t dyn_smem[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dyn_smem) + 1023) & ~uintptr_t(1023));

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&conv_bar[s], kTfConvWarps);
            mbar_init(&empty_bar[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull_bar[a], 1);
            mbar_init(&tempty_bar[a], kTcEpiWarps);
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
    const int KB = (K + kTfBK - 1) / kTfBK;
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
                    mbar_arrive_expect_tx(&full_bar[stage], Cfg::kLoadBytes);
                    tma_load_2d(sa, ma, &full_bar[stage], kb * kTfBK, row0);
                    tma_load_3d(sb, mb, &full_bar[stage], kb * kTfBK, n0, widx);
                    last_parity[stage] = int(phase);
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
            }
            for (int s = 0; s < STAGES; ++s) {
                if (last_parity[s] < 0) continue;
                mbar_wait_drain(&full_bar[s], uint32_t(last_parity[s]));
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------- MMA issuer: lo*hi, hi*lo, hi*hi per K step ----------------
            constexpr uint32_t idesc = idesc_tf32_f32(kTcBM, BN);
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
                    if (!mbar_wait(&conv_bar[stage], phase, abort_p)) { ok = false; break; }
                    tc_fence_after();
                    const uint8_t* sa = smem + size_t(stage) * Cfg::kStageBytes;
                    const uint64_t ahi = sdesc_kmajor_sw128(smem_u32(sa));
                    const uint64_t bhi = sdesc_kmajor_sw128(smem_u32(sa + Cfg::kABytes));
                    const uint64_t alo = sdesc_kmajor_sw128(smem_u32(sa + Cfg::kLoadBytes));
                    const uint64_t blo = sdesc_kmajor_sw128(smem_u32(sa + Cfg::kLoadBytes + Cfg::kABytes));
#pragma unroll
                    for (int kk = 0; kk < kTfBK / 8; ++kk) {   // K = 8 per tf32 MMA = 32 B
                        const uint64_t o = uint64_t(2 * kk);
                        umma_tf32(d_tmem, alo + o, bhi + o, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
                        umma_tf32(d_tmem, ahi + o, blo + o, idesc, 1u);
                        umma_tf32(d_tmem, ahi + o, bhi + o, idesc, 1u);
                    }
                    umma_commit(&empty_bar[stage]);
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                umma_commit(&tfull_bar[acc]);
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1u;
            }
            umma_commit(&drain_bar);
            mbar_wait_drain(&drain_bar, 0);
        }
    } else if (warp >= 2 + kTcEpiWarps) {
        // ---------------- converters (warps 10..17) ----------------
        const int ctid = threadIdx.x - (64 + 32 * kTcEpiWarps);   // 0..255
        constexpr int kVec = int(Cfg::kLoadBytes / 16);           // float4s per stage
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
            for (int kb = 0; kb < KB; ++kb) {
                if (!__all_sync(0xffffffffu, mbar_wait(&full_bar[stage], phase, abort_p))) { ok = false; break; }
                float4* hi = reinterpret_cast<float4*>(smem + size_t(stage) * Cfg::kStageBytes);
                float4* lo = reinterpret_cast<float4*>(smem + size_t(stage) * Cfg::kStageBytes + Cfg::kLoadBytes);
#pragma unroll 4
                for (int i = ctid; i < kVec; i += 32 * kTfConvWarps) {
                    const float4 v = hi[i];
                    float4 h, l;
                    h.x = tf32_round(v.x); l.x = v.x - h.x;
                    h.y = tf32_round(v.y); l.y = v.y - h.y;
                    h.z = tf32_round(v.z); l.z = v.z - h.z;
                    h.w = tf32_round(v.w); l.w = v.w - h.w;
                    hi[i] = h;
                    lo[i] = l;
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&conv_bar[stage]);
                if (++stage == STAGES) { stage = 0; phase ^= 1u; }
            }
        }
    } else {
        // ---------------- epilogue (warps 2..9) ----------------
        const int etid = threadIdx.x - 64;   // 0..255
        const int q = warp & 3;
        const int half = (warp - 2) >> 2;
        int acc = 0;
        uint32_t acc_phase = 0;
        bool failed = false;
        for (int t = blockIdx.x; t < total; t += gridDim.x) {
            if (named_bar_red_or(1, 32 * kTcEpiWarps, failed || *abort_p)) break;
            const TileCoord tc = decode_tile(tt, G, t);
            const bool shared_g = tc.e >= E;
            const int rows = tt.rows[tc.e];
            const int r_in = tc.mt * kTcBM + q * 32 + lane;
            const bool valid = r_in < rows;
            const size_t grow = size_t(tt.crow[tc.e]) + r_in;
            const size_t crow = (out_rows != nullptr && valid && !shared_g) ? size_t(out_rows[grow]) : grow;
            const int n0 = tc.nt * BN;
            float g = 1.f;
            if (MODE == kFc2Gate && row_gate != nullptr && valid && !shared_g) g = row_gate[grow];
            const float* bb = shared_g ? bias2 + size_t(tc.e - E) * N : bias + size_t(tc.e) * N;
            for (int i = etid; i < BN; i += 32 * kTcEpiWarps) sbias[i] = (n0 + i < N) ? bb[n0 + i] : 0.f;
            named_bar_sync(1, 32 * kTcEpiWarps);
            if (!__all_sync(0xffffffffu, mbar_wait(&tfull_bar[acc], acc_phase, abort_p))) {
                failed = true;
                continue;
            }
            tc_fence_after();
#pragma unroll 1
            for (int c = half; c < BN / 32; c += 2) {
                uint32_t r[32];
                __syncwarp();
                tmem_ld_32x32b_x32(tmem_base + (uint32_t(q * 32) << 16) + uint32_t(acc * BN + c * 32), r);
                tmem_ld_wait();
                const int nb = n0 + c * 32;
                if (!valid || nb >= N) continue;
                float* cp = C + crow * N + nb;
#pragma unroll
                for (int v = 0; v < 8; ++v) {
                    if (nb + v * 4 >= N) break;
                    float o[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const float cval = __uint_as_float(r[v * 4 + i]) + sbias[c * 32 + v * 4 + i];
                        o[i] = (MODE == kFc1Gelu) ? gelu_erf(cval) : g * cval;
                    }
                    *reinterpret_cast<float4*>(cp + v * 4) = make_float4(o[0], o[1], o[2], o[3]);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty_bar[acc]);
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1u;
        }
    }

    __syncthreads();
    ffn_clock_mark(clock_on, MODE, 2);
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, Cfg::kTmemCols);
    }
}

}  // namespace moe
