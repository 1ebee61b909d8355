// Step 1 of the layer: the top-k softmax router (cookbook notebook "Mixture-
// of-experts and expert parallelism", section "Top-k router").
//
// Two kernels compute the same thing:
//  * router_tc_kernel (bf16): the logits tile [128 tokens x E] is one
//    tcgen05.mma chain into tensor memory; each epilogue thread then owns one
//    token's logits row (online softmax, register top-k).
//  * router_topk_kernel (fp32 and the fallback-free fp32 path): fp32
//    register-tiled logits over K chunks staged in shared memory, one warp
//    per token for softmax and a k-round warp argmax.
// Both select by logit, largest first, an exact tie going to the lower
// expert index, and both can emit, per token tile, the expert histogram of
// the chosen experts and the per-expert probability sums (used by the
// dispatch scan and the Switch auxiliary loss) without atomics on floats.
#pragma once

#include "common.cuh"

namespace moe {

constexpr int kRouterTM = 32;        // tokens per CTA
constexpr int kRouterKC = 32;        // K chunk staged in shared memory
constexpr int kRouterThreads = 256;  // 16 x 16 thread grid
constexpr int kRouterLd = kRouterKC + 4;

template <int EP>
constexpr size_t router_smem_bytes() {
    return sizeof(float) * (size_t(kRouterTM) * kRouterLd + size_t(EP) * kRouterLd +
                            size_t(kRouterTM) * (EP + 1) + size_t(kRouterThreads / 32) * EP);
}

// load 4 consecutive elements as fp32 (16-byte aligned for f32, 8 for bf16)
__device__ __forceinline__ float4 load4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ float4 load4(const __nv_bfloat16* p) {
    uint2 v = *reinterpret_cast<const uint2*>(p);
    return make_float4(bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y));
}

// EP: expert count padded to a multiple of 16 (16..256)
// prob_sum:  [E], accumulated with one atomicAdd per CTA and expert (caller zeroes it), or
// psum_part: [gridDim.x][E] per-CTA sums (deterministic), and
// hist:      [gridDim.x][E] per-CTA counts of the chosen experts; each may be null.
// F > 0: the token's next F experts in the same order (its fallback experts
// for overflow rerouting) go to fb_idx / fb_gate [T, F]; hist counts only
// the first k.
template <typename Tin, int EP>
__global__ void __launch_bounds__(kRouterThreads)
router_topk_kernel(const Tin* __restrict__ x, const Tin* __restrict__ wr, const float* __restrict__ bias,
                   int T, int d, int E, int k, int32_t* __restrict__ topk_idx, float* __restrict__ topk_gate,
                   float* __restrict__ prob_sum, float* __restrict__ psum_part, int32_t* __restrict__ hist,
                   int F, int32_t* __restrict__ fb_idx, float* __restrict__ fb_gate) {
    constexpr int EPT = EP / 16;          // experts per thread
    constexpr int NV = (EP + 31) / 32;    // expert values per lane in the softmax
    extern __shared__ __align__(16) float smem[];
    float* xs = smem;                                   // [TM][Ld]
    float* ws = xs + kRouterTM * kRouterLd;             // [EP][Ld]
    float* lg = ws + EP * kRouterLd;                    // [TM][EP+1]
    float* red = lg + kRouterTM * (EP + 1);             // [8][EP]
    __shared__ int s_hist[EP];
    for (int e = threadIdx.x; e < EP; e += kRouterThreads) s_hist[e] = 0;

    const int tid = threadIdx.x;
    const int tx = tid & 15, ty = tid >> 4;
    const int t0 = blockIdx.x * kRouterTM;

    pdl_wait();
    pdl_release();
    float acc[2][EPT];
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
        for (int c = 0; c < EPT; ++c) acc[r][c] = 0.f;

    for (int k0 = 0; k0 < d; k0 += kRouterKC) {
        // stage x chunk: 32 tokens x 32 k = 256 vectors of 4
        {
            const int row = tid >> 3, col = (tid & 7) * 4;
            const int t = t0 + row, kk = k0 + col;
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (t < T && kk < d) v = load4(x + size_t(t) * d + kk);
            *reinterpret_cast<float4*>(xs + row * kRouterLd + col) = v;
        }
        for (int v = tid; v < EP * 8; v += kRouterThreads) {
            const int row = v >> 3, col = (v & 7) * 4;
            const int kk = k0 + col;
            float4 w4 = make_float4(0.f, 0.f, 0.f, 0.f);
            if (row < E && kk < d) w4 = load4(wr + size_t(row) * d + kk);
            *reinterpret_cast<float4*>(ws + row * kRouterLd + col) = w4;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < kRouterKC; kk += 4) {
            const float4 a0 = *reinterpret_cast<const float4*>(xs + ty * kRouterLd + kk);
            const float4 a1 = *reinterpret_cast<const float4*>(xs + (ty + 16) * kRouterLd + kk);
#pragma unroll
            for (int c = 0; c < EPT; ++c) {
                const float4 b = *reinterpret_cast<const float4*>(ws + (tx + 16 * c) * kRouterLd + kk);
                acc[0][c] = fmaf(a0.x, b.x, acc[0][c]);
                acc[0][c] = fmaf(a0.y, b.y, acc[0][c]);
                acc[0][c] = fmaf(a0.z, b.z, acc[0][c]);
                acc[0][c] = fmaf(a0.w, b.w, acc[0][c]);
                acc[1][c] = fmaf(a1.x, b.x, acc[1][c]);
                acc[1][c] = fmaf(a1.y, b.y, acc[1][c]);
                acc[1][c] = fmaf(a1.z, b.z, acc[1][c]);
                acc[1][c] = fmaf(a1.w, b.w, acc[1][c]);
            }
        }
        __syncthreads();
    }

#pragma unroll
    for (int c = 0; c < EPT; ++c) {
        const int e = tx + 16 * c;
        const float b = (bias != nullptr && e < E) ? bias[e] : 0.f;
        lg[ty * (EP + 1) + e] = acc[0][c] + b;
        lg[(ty + 16) * (EP + 1) + e] = acc[1][c] + b;
    }
    __syncthreads();

    const int warp = tid >> 5, lane = tid & 31;
    float psum[NV];
#pragma unroll
    for (int c = 0; c < NV; ++c) psum[c] = 0.f;

    for (int r = warp; r < kRouterTM; r += kRouterThreads / 32) {
        const int t = t0 + r;
        if (t >= T) break;
        float v[NV];
        float m = -INFINITY;
#pragma unroll
        for (int c = 0; c < NV; ++c) {
            const int e = lane + 32 * c;
            float l = (e < E) ? lg[r * (EP + 1) + e] : -INFINITY;
            if (l != l) l = -INFINITY;   // NaN never wins a slot
            v[c] = l;
            m = fmaxf(m, l);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        float s = 0.f;
        float p[NV];
#pragma unroll
        for (int c = 0; c < NV; ++c) {
            p[c] = (lane + 32 * c < E) ? expf(v[c] - m) : 0.f;
            s += p[c];
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        const float inv = 1.0f / s;
#pragma unroll
        for (int c = 0; c < NV; ++c) psum[c] += p[c] * inv;

        uint32_t taken = 0;
        for (int j = 0; j < k + F; ++j) {
            float bv = -INFINITY;
            int be = 0x7fffffff;
#pragma unroll
            for (int c = 0; c < NV; ++c) {
                const int e = lane + 32 * c;
                if (e < E && !((taken >> c) & 1u) && (v[c] > bv || (v[c] == bv && e < be))) {
                    bv = v[c];
                    be = e;
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
                const int oe = __shfl_xor_sync(0xffffffffu, be, o);
                if (ov > bv || (ov == bv && oe < be)) {
                    bv = ov;
                    be = oe;
                }
            }
            if ((be & 31) == lane) taken |= 1u << (be >> 5);
            if (lane == 0) {
                if (j < k) {
                    topk_idx[size_t(t) * k + j] = be;
                    topk_gate[size_t(t) * k + j] = expf(bv - m) * inv;
                    atomicAdd(&s_hist[be], 1);
                } else {
                    fb_idx[size_t(t) * F + (j - k)] = be;
                    fb_gate[size_t(t) * F + (j - k)] = expf(bv - m) * inv;
                }
            }
        }
    }

#pragma unroll
    for (int c = 0; c < NV; ++c) {
        const int e = lane + 32 * c;
        if (e < EP) red[warp * EP + e] = psum[c];
    }
    __syncthreads();
    for (int e = tid; e < E; e += kRouterThreads) {
        float tot = 0.f;
#pragma unroll
        for (int w = 0; w < kRouterThreads / 32; ++w) tot += red[w * EP + e];
        if (psum_part != nullptr) psum_part[size_t(blockIdx.x) * E + e] = tot;
        else if (prob_sum != nullptr) atomicAdd(prob_sum + e, tot);
        if (hist != nullptr) hist[size_t(blockIdx.x) * E + e] = s_hist[e];
    }
}

// ===========================================================================
// bf16 router on the tensor cores.  One CTA per 128-token tile, 320 threads:
//   warp 0      TMA producer: x tile rows [t0, t0+128) and W_r, 64 columns of
//               K per stage (128B swizzle; rows past T and experts past E
//               are zero-filled by the tensor maps); as many stages as fit
//   warp 1      TMEM allocator and MMA issuer: logits[128 x EP] in fp32
//   warps 2..9  epilogue, two warps per TMEM lane quarter, thread = token:
//               for E <= 64 each of the two takes one 32-expert chunk of its
//               32 tokens' logits (+ bias from shared memory), its local max,
//               exponentials, sum and top-k; the two exchange those through
//               shared memory and merge them (softmax of the whole row, top-k
//               with ties to the lower index); then each warp's share of the
//               per-expert probability column sums (a shared-memory transpose,
//               fixed summation order) and the expert histogram.  For E > 64
//               warps 2..5 make two passes over all the chunks.
// Once the last MMA has completed the pipeline stages are free, and the
// epilogue uses them as scratch (the exchange records and the transposes).
// ===========================================================================
constexpr int kRtBM = 128;
constexpr int kRtEpiWarps = 8;
constexpr int kRtThreads = 64 + 32 * kRtEpiWarps;
// dynamic shared memory the stages may take, leaving room for the static
// arrays (< 4 KB) below the 227 KB a CTA can have
constexpr size_t kRtDynBudget = 227u * 1024u - 4096u;

// SPLIT = 2: the two CTAs of a cluster split a tile's K stages; the
// second sends its partial logits [128 x EP] (fp32) into the first's
// shared memory, past the stages
template <int EP, int SPLIT = 1>
struct RtCfg {
    static constexpr uint32_t kABytes = kRtBM * 64 * 2;
    static constexpr uint32_t kBBytes = EP * 64 * 2;
    static constexpr uint32_t kStageBytes = kABytes + kBBytes;
    static constexpr uint32_t kPartBytes = SPLIT == 2 ? kRtBM * EP * 4 : 0;
    static constexpr int kFit = int((kRtDynBudget - 1024 - kPartBytes) / kStageBytes);
    static constexpr int kStages = kFit < 12 ? kFit : 12;
    static constexpr uint32_t kTmemCols = EP < 32 ? 32 : EP;
    static constexpr size_t kPartOffset = size_t(kStages) * kStageBytes;
    static constexpr size_t kSmemBytes = kPartOffset + kPartBytes + 1024;
    static_assert(kStages >= 4, "at least four stages");
    static_assert(SPLIT == 1 || EP <= 64, "K split only with one or two logit chunks");
};

// shared::cluster address of the same shared-memory location in CTA `rank`
__device__ __forceinline__ uint32_t mapa_rank(uint32_t smem_addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr), "r"(rank));
    return r;
}
// 16-byte store to a shared::cluster address (another CTA's shared memory)
__device__ __forceinline__ void st_cluster_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared::cluster.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d)
                 : "memory");
}

// per-row record one epilogue warp hands to its partner (E <= 64)
template <int KMAX>
struct RtRec {
    float m, s;          // chunk max logit, sum of exp(logit - m)
    float v[KMAX];       // chunk top-KMAX logits, largest first
    int ix[KMAX];        // their expert indices (ties: lower index first)
};

// KMAX >= k + F: the selection also yields the F fallback experts (fb_idx /
// fb_gate [T, F]), as in router_topk_kernel.
// SPLIT = 2 (clusters of two CTAs, grid = 2 x tiles): CTA rank r of tile
// blockIdx.x / 2 takes K stages [r * KB/2, (r+1) * KB/2) (the second half
// also the remainder); rank 1's epilogue warps store their partial logits
// into rank 0's shared memory (distributed shared memory), one cluster
// barrier that every thread of both CTAs reaches, then rank 0 adds them
// and runs the epilogue below on the whole tile; rank 1 writes nothing else.
template <int EP, int KMAX, int SPLIT>
__global__ void __launch_bounds__(kRtThreads, 1)
router_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                 const float* __restrict__ bias, int T, int d, int E, int k, int32_t* __restrict__ topk_idx,
                 float* __restrict__ topk_gate, float* __restrict__ prob_sum, float* __restrict__ psum_part,
                 int32_t* __restrict__ hist, int F, int32_t* __restrict__ fb_idx, float* __restrict__ fb_gate) {
    using Cfg = RtCfg<EP, SPLIT>;
    constexpr int S = Cfg::kStages;
    constexpr int NCH = (EP + 31) / 32;   // 32-column TMEM chunks
    __shared__ __align__(8) uint64_t full_bar[S], empty_bar[S], done_bar;
    __shared__ uint32_t tmem_slot;
    __shared__ int abort_flag;
    __shared__ int s_hist[EP];
    __shared__ float s_bias[EP];
    __shared__ float s_col[4][NCH * 32];     // per lane quarter: column sums of the probabilities
    extern __shared__ uint8_t dyn_smem[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dyn_smem) + 1023) & ~uintptr_t(1023));

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int i = 0; i < S; ++i) {
            mbar_init(&full_bar[i], 1);
            mbar_init(&empty_bar[i], 1);
        }
        mbar_init(&done_bar, 1);
        abort_flag = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tmX);
        tma_prefetch_desc(&tmW);
    }
    for (int e = threadIdx.x; e < EP; e += kRtThreads) s_hist[e] = 0;
    for (int i = threadIdx.x; i < 4 * NCH * 32; i += kRtThreads) (&s_col[0][0])[i] = 0.f;
    if (warp == 1) {
        tmem_alloc(&tmem_slot, Cfg::kTmemCols);
        tmem_relinquish();
        tc_fence_before();
    }
    __syncthreads();
    tc_fence_after();
    pdl_wait();
    pdl_release();
    const uint32_t tmem_base = tmem_slot;
    const int KB = (d + 63) / 64;
    const uint32_t rank = SPLIT == 2 ? cluster_ctarank() : 0u;
    const int tile = SPLIT == 2 ? int(blockIdx.x >> 1) : int(blockIdx.x);
    const int kb_lo = SPLIT == 2 ? int(rank) * (KB / 2) : 0;
    const int kb_hi = (SPLIT == 2 && rank == 0) ? KB / 2 : KB;
    const int t0 = tile * kRtBM;
    volatile int* abort_p = &abort_flag;

    if (warp == 0) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int last_parity[S];
            for (int i = 0; i < S; ++i) last_parity[i] = -1;
            for (int kb = kb_lo; kb < kb_hi; ++kb) {
                if (!mbar_wait(&empty_bar[stage], phase ^ 1u, abort_p)) break;
                uint8_t* sa = smem + size_t(stage) * Cfg::kStageBytes;
                mbar_arrive_expect_tx(&full_bar[stage], Cfg::kStageBytes);
                tma_load_2d(sa, &tmX, &full_bar[stage], kb * 64, t0);
                tma_load_2d(sa + Cfg::kABytes, &tmW, &full_bar[stage], kb * 64, 0);
                last_parity[stage] = int(phase);
                if (++stage == S) { stage = 0; phase ^= 1u; }
            }
            for (int i = 0; i < S; ++i)
                if (last_parity[i] >= 0) mbar_wait_drain(&full_bar[i], uint32_t(last_parity[i]));
        }
        if constexpr (SPLIT == 2) cluster_sync();
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(kRtBM, EP);
            int stage = 0;
            uint32_t phase = 0;
            for (int kb = kb_lo; kb < kb_hi; ++kb) {
                if (!mbar_wait(&full_bar[stage], phase, abort_p)) break;
                tc_fence_after();
                const uint8_t* sa = smem + size_t(stage) * Cfg::kStageBytes;
                const uint64_t adesc = sdesc_kmajor_sw128(smem_u32(sa));
                const uint64_t bdesc = sdesc_kmajor_sw128(smem_u32(sa + Cfg::kABytes));
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    umma_f16(tmem_base, adesc + uint64_t(2 * kk), bdesc + uint64_t(2 * kk), idesc,
                             (kb > kb_lo || kk > 0) ? 1u : 0u);
                umma_commit(&empty_bar[stage]);
                if (++stage == S) { stage = 0; phase ^= 1u; }
            }
            umma_commit(&done_bar);   // tracks every MMA issued above
            // TMEM is released only after those MMAs complete (bounded wait)
            mbar_wait_drain(&done_bar, 0);
        }
        if constexpr (SPLIT == 2) cluster_sync();
    } else {
        const int etid = threadIdx.x - 64;    // 0..255
        const int q = warp & 3;               // TMEM lane quarter
        const int c = (warp - 2) >> 2;        // 0: warps 2..5, 1: warps 6..9
        const int row = q * 32 + lane;
        const int t = t0 + row;
        const bool valid = t < T;
        for (int e = etid; e < EP; e += 32 * kRtEpiWarps) s_bias[e] = (bias != nullptr && e < E) ? bias[e] : 0.f;
        named_bar_sync(1, 32 * kRtEpiWarps);   // the bias is visible
        const bool ok = mbar_wait(&done_bar, 0, abort_p);
        tc_fence_after();
        // scratch in the (now idle) pipeline stages: per warp a 32 x 33
        // transpose tile, then the exchange records [2][128]
        float* tr = reinterpret_cast<float*>(smem) + (warp - 2) * (32 * 33);
        RtRec<KMAX>* rec = reinterpret_cast<RtRec<KMAX>*>(smem + size_t(kRtEpiWarps) * 32 * 33 * sizeof(float));
        if constexpr (NCH <= 2) {
            // ---- one 32-expert chunk per warp ----
            uint32_t r[32];
            if (c < NCH) {
                __syncwarp();
                tmem_ld_32x32b_x32(tmem_base + (uint32_t(q * 32) << 16) + uint32_t(c * 32), r);
                tmem_ld_wait();
            }
            if constexpr (SPLIT == 2) {
                // the K split: rank 1 hands its partial logits to rank 0
                constexpr int kCols = EP < 32 ? EP : 32;   // valid columns of a chunk
                float* part = reinterpret_cast<float*>(smem + Cfg::kPartOffset) + size_t(row) * EP + c * 32;
                if (rank == 1 && c < NCH) {
                    const uint32_t remote = mapa_rank(smem_u32(part), 0);
#pragma unroll
                    for (int i = 0; i < kCols; i += 4)
                        st_cluster_v4(remote + uint32_t(i) * 4u, r[i], r[i + 1], r[i + 2], r[i + 3]);
                }
                cluster_sync();   // every thread of both CTAs passes here once
                if (rank == 0 && c < NCH) {
#pragma unroll
                    for (int i = 0; i < kCols; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) + part[i]);
                }
            }
          if (SPLIT == 1 || rank == 0) {
            float l[32];
            float m = -INFINITY;
            if (c < NCH) {
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int e = c * 32 + i;
                    float v = (e < E && ok) ? __uint_as_float(r[i]) + s_bias[e] : -INFINITY;
                    if (v != v) v = -INFINITY;
                    l[i] = v;
                    m = fmaxf(m, v);
                }
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) l[i] = -INFINITY;
            }
            // exponentials relative to the chunk max and their sum
            float ex[32];
            float ps[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                ex[i] = (l[i] == -INFINITY) ? 0.f : __expf(l[i] - m);
                ps[i & 3] += ex[i];
            }
            const float sc = (ps[0] + ps[1]) + (ps[2] + ps[3]);
            // chunk top-KMAX by logit (largest first; a later equal value does
            // not displace an earlier one, so ties keep the lower index)
            float tv[KMAX];
            int ti[KMAX];
#pragma unroll
            for (int j = 0; j < KMAX; ++j) {
                tv[j] = -INFINITY;
                ti[j] = 0x7fffffff;
            }
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                float v = l[i];
                int ix = c * 32 + i;
                if (v == -INFINITY || !(v > tv[KMAX - 1])) continue;
#pragma unroll
                for (int j = 0; j < KMAX; ++j) {
                    if (v > tv[j]) {
                        const float tf = tv[j];
                        tv[j] = v;
                        v = tf;
                        const int tix = ti[j];
                        ti[j] = ix;
                        ix = tix;
                    }
                }
            }
            // exchange with the partner warp (same lane quarter, other chunk)
            {
                RtRec<KMAX>& mine = rec[c * kRtBM + row];
                mine.m = m;
                mine.s = sc;
#pragma unroll
                for (int j = 0; j < KMAX; ++j) {
                    mine.v[j] = tv[j];
                    mine.ix[j] = ti[j];
                }
            }
            named_bar_sync(1, 32 * kRtEpiWarps);
            const RtRec<KMAX>& other = rec[(1 - c) * kRtBM + row];
            const float mo = other.m;
            const float M = fmaxf(m, mo);
            const float f_mine = (m == -INFINITY) ? 0.f : __expf(m - M);
            const float f_other = (mo == -INFINITY) ? 0.f : __expf(mo - M);
            const float Ssum = sc * f_mine + other.s * f_other;
            const float inv = Ssum > 0.f ? 1.0f / Ssum : 0.f;
            if (c == 0 && valid && ok) {
                // merge the two sorted lists: chunk 0 holds the lower indices,
                // so on equal logits it goes first (the heads are compared and
                // the taken list shifted, keeping every index static)
                float ov[KMAX];
                int oi[KMAX];
#pragma unroll
                for (int j = 0; j < KMAX; ++j) {
                    ov[j] = other.v[j];
                    oi[j] = other.ix[j];
                }
#pragma unroll
                for (int j = 0; j < KMAX; ++j) {
                    if (j < k + F) {
                        const bool take_a = tv[0] >= ov[0];
                        const float v = take_a ? tv[0] : ov[0];
                        int e = take_a ? ti[0] : oi[0];
#pragma unroll
                        for (int i = 0; i + 1 < KMAX; ++i) {
                            tv[i] = take_a ? tv[i + 1] : tv[i];
                            ti[i] = take_a ? ti[i + 1] : ti[i];
                            ov[i] = take_a ? ov[i] : ov[i + 1];
                            oi[i] = take_a ? oi[i] : oi[i + 1];
                        }
                        if (take_a) {
                            tv[KMAX - 1] = -INFINITY;
                            ti[KMAX - 1] = 0x7fffffff;
                        } else {
                            ov[KMAX - 1] = -INFINITY;
                            oi[KMAX - 1] = 0x7fffffff;
                        }
                        if (e >= E) e = j;   // fewer finite logits than k + F (a NaN row): valid indices
                        const float g = (v == -INFINITY) ? 0.f : __expf(v - M) * inv;
                        if (j < k) {
                            topk_idx[size_t(t) * k + j] = e;
                            topk_gate[size_t(t) * k + j] = g;
                            atomicAdd(&s_hist[e], 1);
                        } else {
                            fb_idx[size_t(t) * F + (j - k)] = e;
                            fb_gate[size_t(t) * F + (j - k)] = g;
                        }
                    }
                }
            }
            if ((prob_sum != nullptr || psum_part != nullptr) && c < NCH) {
                const float scale = f_mine * inv;
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    tr[lane * 33 + i] = (valid && ok && c * 32 + i < E) ? ex[i] * scale : 0.f;
                __syncwarp();
                float cs = 0.f;
#pragma unroll
                for (int i = 0; i < 32; ++i) cs += tr[i * 33 + lane];
                s_col[q][c * 32 + lane] = cs;
            }
          }
        } else if (c == 0) {
            // ---- E > 64: warps 2..5, two passes over all the chunks ----
            float m = -INFINITY, ssum = 0.f;
            float tv[KMAX];
            int ti[KMAX];
#pragma unroll
            for (int j = 0; j < KMAX; ++j) {
                tv[j] = -INFINITY;
                ti[j] = 0x7fffffff;
            }
            // pass 1: online softmax statistics and top-k over the logits row
#pragma unroll 1
            for (int ch = 0; ch < NCH; ++ch) {
                uint32_t r[32];
                __syncwarp();
                tmem_ld_32x32b_x32(tmem_base + (uint32_t(q * 32) << 16) + uint32_t(ch * 32), r);
                tmem_ld_wait();
                float l[32];
                float cm = -INFINITY;
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int e = ch * 32 + i;
                    float v = (e < E && ok) ? __uint_as_float(r[i]) + s_bias[e] : -INFINITY;
                    if (v != v) v = -INFINITY;
                    l[i] = v;
                    cm = fmaxf(cm, v);
                }
                const float mn = fmaxf(m, cm);
                if (mn != -INFINITY) {
                    float acc = (m == -INFINITY) ? 0.f : ssum * expf(m - mn);
#pragma unroll
                    for (int i = 0; i < 32; ++i) acc += (l[i] == -INFINITY) ? 0.f : expf(l[i] - mn);
                    ssum = acc;
                    m = mn;
                }
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    float v = l[i];
                    int ix = ch * 32 + i;
                    if (v == -INFINITY || !(v > tv[KMAX - 1])) continue;
#pragma unroll
                    for (int j = 0; j < KMAX; ++j) {
                        if (v > tv[j]) {
                            const float tf = tv[j];
                            tv[j] = v;
                            v = tf;
                            const int tix = ti[j];
                            ti[j] = ix;
                            ix = tix;
                        }
                    }
                }
            }
            const float inv = 1.0f / ssum;
            if (valid && ok) {
#pragma unroll
                for (int j = 0; j < KMAX; ++j) {
                    if (j < k + F) {
                        // fewer than k + F finite logits cannot happen for k + F <= E with finite inputs;
                        // guard so an all-NaN row still yields valid, distinct indices
                        int e = ti[j];
                        if (e >= E) e = j;
                        const float g = (tv[j] == -INFINITY) ? 0.f : expf(tv[j] - m) * inv;
                        if (j < k) {
                            topk_idx[size_t(t) * k + j] = e;
                            topk_gate[size_t(t) * k + j] = g;
                            atomicAdd(&s_hist[e], 1);
                        } else {
                            fb_idx[size_t(t) * F + (j - k)] = e;
                            fb_gate[size_t(t) * F + (j - k)] = g;
                        }
                    }
                }
            }
            // pass 2: per-expert sums of this tile's probabilities (fixed order)
            if (prob_sum != nullptr || psum_part != nullptr) {
#pragma unroll 1
                for (int ch = 0; ch < NCH; ++ch) {
                    uint32_t r[32];
                    __syncwarp();
                    tmem_ld_32x32b_x32(tmem_base + (uint32_t(q * 32) << 16) + uint32_t(ch * 32), r);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int e = ch * 32 + i;
                        float p = 0.f;
                        if (valid && ok && e < E) {
                            float v = __uint_as_float(r[i]) + s_bias[e];
                            p = (v != v) ? 0.f : expf(v - m) * inv;
                        }
                        tr[lane * 33 + i] = p;
                    }
                    __syncwarp();
                    float cs = 0.f;
#pragma unroll
                    for (int i = 0; i < 32; ++i) cs += tr[i * 33 + lane];
                    s_col[q][ch * 32 + lane] = cs;
                    __syncwarp();
                }
            }
        }
        tc_fence_before();
    }
    __syncthreads();
    if (SPLIT == 1 || rank == 0) {
        for (int e = threadIdx.x; e < E; e += kRtThreads) {
            const float tot = ((s_col[0][e] + s_col[1][e]) + s_col[2][e]) + s_col[3][e];
            if (psum_part != nullptr) psum_part[size_t(tile) * E + e] = tot;
            else if (prob_sum != nullptr) atomicAdd(prob_sum + e, tot);
            if (hist != nullptr) hist[size_t(tile) * E + e] = s_hist[e];
        }
    }
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, Cfg::kTmemCols);
    }
}

}  // namespace moe
