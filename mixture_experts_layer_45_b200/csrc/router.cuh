// Step 1 of the layer: the top-k softmax router (cookbook notebook "Mixture-
// of-experts and expert parallelism", section "Top-k router").
//
// One CTA owns kRouterTM tokens.  The logits tile [tokens x experts] is an
// fp32 register-tiled product over K chunks staged in shared memory; then
// one warp per token does the max-subtracted softmax, the k-round warp
// argmax (ties -> lower expert index) and the per-expert probability sums
// used by the Switch auxiliary loss.
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
template <typename Tin, int EP>
__global__ void __launch_bounds__(kRouterThreads)
router_topk_kernel(const Tin* __restrict__ x, const Tin* __restrict__ wr, const float* __restrict__ bias,
                   int T, int d, int E, int k, int32_t* __restrict__ topk_idx, float* __restrict__ topk_gate,
                   float* __restrict__ prob_sum) {
    constexpr int EPT = EP / 16;          // experts per thread
    constexpr int NV = (EP + 31) / 32;    // expert values per lane in the softmax
    extern __shared__ __align__(16) float smem[];
    float* xs = smem;                                   // [TM][Ld]
    float* ws = xs + kRouterTM * kRouterLd;             // [EP][Ld]
    float* lg = ws + EP * kRouterLd;                    // [TM][EP+1]
    float* red = lg + kRouterTM * (EP + 1);             // [8][EP]

    const int tid = threadIdx.x;
    const int tx = tid & 15, ty = tid >> 4;
    const int t0 = blockIdx.x * kRouterTM;

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
        for (int j = 0; j < k; ++j) {
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
                topk_idx[size_t(t) * k + j] = be;
                topk_gate[size_t(t) * k + j] = expf(bv - m) * inv;
            }
        }
    }

    if (prob_sum != nullptr) {
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
            atomicAdd(prob_sum + e, tot);
        }
    }
}

}  // namespace moe
