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
// Each fp32 operand v is split into a TF32 part hi and lo = v - hi (exact in
// fp32): for the activations A hi = v rounded to nearest on the 13 low
// mantissa bits (|lo| <= 2^-11 |hi|); for the weights hi = v truncated to
// its top 19 bits, which is what the tensor cores read of the raw fp32
// value, so the weight tile is used as loaded (|lo| < 2^-10 |hi|).  Then
// A B^T = hi_A hi_B^T + hi_A lo_B^T + lo_A hi_B^T + lo_A lo_B^T and the last
// product, at most about 2^-21 of the result, is dropped.  Each kept
// product is a tcgen05.mma kind::tf32 with fp32 accumulation in tensor
// memory, so the result carries fp32-level error (the split-precision
// scheme of Ootomo & Yokota 2022) at the tensor cores' TF32 rate.
//
// The A operand (the 128 activation rows) goes to the tensor cores from
// tensor memory, the weight operand from shared memory: per K step the
// converters read the landed A tile once and write its hi and lo parts
// straight into the stage's two TMEM operand regions (tcgen05.st), and
// the weight tile gets only a lo tile beside it.  Per stage that moves 128
// KB through shared memory (TMA 32, converter reads 32, weight lo writes
// 16, MMA operand reads 48) for 768 tensor cycles, where staging A's parts
// in shared memory too (and rewriting both hi parts) moved 224 KB.
//
// Warp roles (576 threads):
//   warp 0        TMA producer: raw fp32 A and W tiles, 32 columns (128 B)
//                 of K per stage, 128B swizzle
//   warp 1        TMEM allocator and MMA issuer: 3 MMAs per K step of 8,
//                 A from tensor memory
//   warps 2..9    epilogue, as the bf16 kernel, fp32 stores
//   warps 10..17  converters: for each landed stage, warp w takes TMEM lane
//                 quarter w % 4 and half (w - 10) / 4 of the 32 K columns of
//                 A (lane = row: 16 values from the swizzled tile, split, two
//                 tcgen05.st), then an eighth of the weight tile's lo parts
//                 into the lo tile (same swizzled positions); then
//                 the TMEM stores are waited for and the shared-memory writes
//                 fenced to the async proxy before the stage is released to
//                 the MMA issuer
//
// Tensor memory (512 columns): the two accumulators (BN columns each), then
// per stage A hi (32 columns: one per K element, lane = row) and A lo.
// ===========================================================================
constexpr int kTfBK = 32;            // 32 fp32 = 128 B = one swizzle row
constexpr int kTfConvWarps = 8;
constexpr int kTfThreads = 64 + 32 * kTcEpiWarps + 32 * kTfConvWarps;

template <int BN, int STAGES>
struct TfCfg {
    static constexpr uint32_t kABytes = kTcBM * kTfBK * 4;
    static constexpr uint32_t kBBytes = BN * kTfBK * 4;
    static constexpr uint32_t kLoadBytes = kABytes + kBBytes;        // what TMA brings per stage
    static constexpr uint32_t kStageBytes = kLoadBytes + kBBytes;    // + the weight lo tile
    static constexpr uint32_t kAOpCol = 2 * BN;                      // first TMEM column of the A parts
    static constexpr uint32_t kTmemCols = 512;
    static constexpr size_t kSmemBytes = size_t(STAGES) * kStageBytes + 1024;
    static_assert(2 * BN + STAGES * 2 * kTfBK <= 512, "accumulators and A operand parts fit in TMEM");
    // TMEM column of stage s's A hi (part 0) or lo (part 1)
    __host__ __device__ static constexpr uint32_t a_col(int s, int part) { return kAOpCol + uint32_t(s * 2 + part) * kTfBK; }
};

// D(tmem) (+)= A(tmem) * B(smem)^T, kind::tf32: A's 128 rows in the 128
// lanes, its K elements in consecutive columns
__device__ __forceinline__ void umma_tf32_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc, uint32_t idesc,
                                             uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(tmem_d),
        "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// this warp's lane quarter: lane i writes 16 consecutive 32-bit columns of
// TMEM lane (quarter base + i)
__device__ __forceinline__ void tmem_st_32x32b_x16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// What kind::tf32 reads of an fp32 operand: its top 19 bits (sign, exponent,
// 10 mantissa bits), the low 13 mantissa bits cleared.  (Checked on B200: a
// weight split as raw value plus v - tf32_trunc(v) gives the same error as
// the explicit round-to-nearest split, 2.8e-5 against 2.7e-5 max-norm
// relative on d = 768, ff = 3072; a rounding tensor core would leave an
// error near 2^-11.)
__device__ __forceinline__ float tf32_trunc(float v) { return __uint_as_float(__float_as_uint(v) & 0xFFFFE000u); }

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
                    const uint64_t bhi = sdesc_kmajor_sw128(smem_u32(sa + Cfg::kABytes));
                    const uint64_t blo = sdesc_kmajor_sw128(smem_u32(sa + Cfg::kLoadBytes));
                    const uint32_t ahi = tmem_base + Cfg::a_col(stage, 0);
                    const uint32_t alo = tmem_base + Cfg::a_col(stage, 1);
#pragma unroll
                    for (int kk = 0; kk < kTfBK / 8; ++kk) {   // K = 8 per tf32 MMA: 32 B of B, 8 TMEM columns of A
                        const uint64_t o = uint64_t(2 * kk);
                        const uint32_t c = uint32_t(8 * kk);
                        umma_tf32_ts(d_tmem, alo + c, bhi + o, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
                        umma_tf32_ts(d_tmem, ahi + c, blo + o, idesc, 1u);
                        umma_tf32_ts(d_tmem, ahi + c, bhi + o, idesc, 1u);
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
        const int q = warp & 3;                                   // TMEM lane quarter
        const int hh = (warp - (2 + kTcEpiWarps)) >> 2;           // half of A's 32 K columns
        const int row = q * 32 + lane;                            // A row = TMEM lane
        const uint32_t lane_base = tmem_base + (uint32_t(q * 32) << 16);
        constexpr int kBVec = int(Cfg::kBBytes / 16);             // float4s of the weight tile
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
            for (int kb = 0; kb < KB; ++kb) {
                if (!__all_sync(0xffffffffu, mbar_wait(&full_bar[stage], phase, abort_p))) { ok = false; break; }
                uint8_t* st_base = smem + size_t(stage) * Cfg::kStageBytes;
                // A: row `row`, 16-byte chunks 4*hh .. 4*hh+3 of its 128 bytes
                // (128B swizzle: chunk c of row r sits at chunk c ^ (r & 7))
                uint32_t ahi[16], alo[16];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int c = 4 * hh + j;
                    const float4 v = *reinterpret_cast<const float4*>(st_base + size_t(row) * 128 +
                                                                      size_t((c ^ (row & 7)) << 4));
                    const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const float h = tf32_round(vv[i]);
                        ahi[j * 4 + i] = __float_as_uint(h);
                        alo[j * 4 + i] = __float_as_uint(vv[i] - h);
                    }
                }
                tmem_st_32x32b_x16(lane_base + Cfg::a_col(stage, 0) + uint32_t(16 * hh), ahi);
                tmem_st_32x32b_x16(lane_base + Cfg::a_col(stage, 1) + uint32_t(16 * hh), alo);
                // the weight tile stays as loaded (its hi part is what the
                // tensor cores read of it); its lo part into the stage's lo tile
                const float4* bw = reinterpret_cast<const float4*>(st_base + Cfg::kABytes);
                float4* blo = reinterpret_cast<float4*>(st_base + Cfg::kLoadBytes);
#pragma unroll 4
                for (int i = ctid; i < kBVec; i += 32 * kTfConvWarps) {
                    const float4 v = bw[i];
                    blo[i] = make_float4(v.x - tf32_trunc(v.x), v.y - tf32_trunc(v.y), v.z - tf32_trunc(v.z),
                                         v.w - tf32_trunc(v.w));
                }
                tmem_st_wait();               // this warp's TMEM stores are done
                fence_proxy_async_smem();     // the tensor cores see the shared-memory writes
                tc_fence_before();
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
