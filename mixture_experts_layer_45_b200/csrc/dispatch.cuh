// Step 2 of the layer: dispatch (cookbook notebook "Mixture-of-experts and
// expert parallelism", sections "Capacity factor" and "Dispatch and
// gather").  Groups the T*k assignments by expert, expert e keeping its first
// kept_e = min(count_e, capacity) assignments in token order.
//
// Four launches, none of which lets thread timing decide a position:
//   count    per-chunk expert histograms (shared-memory integer atomics;
//            integer addition commutes, so the counts are exact)
//   scan     per-(chunk, expert) bases, counts, capacity clamp, offsets
//   permute  stable in-chunk ranks from warp match/ballot masks, then
//            perm / slot_of / drop_mask / row_gate
//   gather   xp[row] = x[token of perm[row]], one warp per row, 16-byte copies
#pragma once

#include "common.cuh"

namespace moe {

constexpr int kDispThreads = 256;
constexpr int kDispWarps = kDispThreads / 32;
constexpr int kDispChunk = 2048;                       // assignments per CTA
constexpr int kDispPerWarp = kDispChunk / kDispWarps;  // 256 = 8 rounds of 32

__global__ void __launch_bounds__(kDispThreads)
dispatch_count_kernel(const int32_t* __restrict__ idx, int A, int E, int32_t* __restrict__ hist) {
    pdl_wait();
    pdl_release();
    __shared__ int h[MOE_MAX_EXPERTS];
    for (int e = threadIdx.x; e < E; e += kDispThreads) h[e] = 0;
    __syncthreads();
    const int a0 = blockIdx.x * kDispChunk;
    for (int i = threadIdx.x; i < kDispChunk; i += kDispThreads) {
        const int a = a0 + i;
        if (a >= A) break;
        const int e = idx[a];
        if (e >= 0 && e < E)
            atomicAdd(&h[e], 1);
        else
            set_error(MOE_ERR_BAD_ROUTING);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += kDispThreads) hist[size_t(blockIdx.x) * E + e] = h[e];
}

// One CTA.  base[b][e] = number of expert-e assignments in chunks before b.
__global__ void __launch_bounds__(kDispThreads)
dispatch_scan_kernel(const int32_t* __restrict__ hist, int nblk, int E, int capacity,
                     int32_t* __restrict__ base, int32_t* __restrict__ counts, int32_t* __restrict__ offsets) {
    pdl_wait();
    pdl_release();
    __shared__ int kept[MOE_MAX_EXPERTS];
    for (int e = threadIdx.x; e < E; e += kDispThreads) {
        int run = 0;
        for (int b = 0; b < nblk; ++b) {
            base[size_t(b) * E + e] = run;
            run += hist[size_t(b) * E + e];
        }
        if (counts != nullptr) counts[e] = run;
        kept[e] = capacity < 0 ? run : min(run, capacity);
    }
    __syncthreads();
    if (threadIdx.x < 32) {
        // exclusive scan of kept over experts: lane l owns experts 8l .. 8l+7
        const int lane = threadIdx.x;
        int local[MOE_MAX_EXPERTS / 32];
        int sum = 0;
#pragma unroll
        for (int i = 0; i < MOE_MAX_EXPERTS / 32; ++i) {
            const int e = lane * (MOE_MAX_EXPERTS / 32) + i;
            local[i] = e < E ? kept[e] : 0;
            sum += local[i];
        }
        int incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        int run = incl - sum;
#pragma unroll
        for (int i = 0; i < MOE_MAX_EXPERTS / 32; ++i) {
            const int e = lane * (MOE_MAX_EXPERTS / 32) + i;
            if (e < E) offsets[e] = run;
            run += local[i];
        }
        if (lane == 31) offsets[E] = incl;
    }
}

__global__ void __launch_bounds__(kDispThreads)
dispatch_permute_kernel(const int32_t* __restrict__ idx, const float* __restrict__ gate, int A, int E,
                        const int32_t* __restrict__ base, const int32_t* __restrict__ offsets,
                        int32_t* __restrict__ perm, int32_t* __restrict__ slot_of, uint8_t* __restrict__ drop_mask,
                        float* __restrict__ row_gate) {
    pdl_wait();
    pdl_release();
    __shared__ int wcnt[kDispWarps][MOE_MAX_EXPERTS];
    __shared__ int off_s[MOE_MAX_EXPERTS + 1];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    for (int i = tid; i < kDispWarps * MOE_MAX_EXPERTS; i += kDispThreads) (&wcnt[0][0])[i] = 0;
    for (int e = tid; e <= E; e += kDispThreads) off_s[e] = offsets[e];
    __syncthreads();

    const uint32_t lt_mask = (1u << lane) - 1u;
    const int a_warp = blockIdx.x * kDispChunk + warp * kDispPerWarp;
    constexpr int kRounds = kDispPerWarp / 32;
    int ex[kRounds], rank[kRounds];
#pragma unroll
    for (int r = 0; r < kRounds; ++r) {
        const int a = a_warp + r * 32 + lane;
        int e = (a < A) ? idx[a] : -1;
        if (e >= E) e = -1;
        if (e < -1) e = -1;
        const uint32_t peers = __match_any_sync(0xffffffffu, e);
        const int local = __popc(peers & lt_mask);
        rank[r] = (e >= 0) ? wcnt[warp][e] + local : 0;
        __syncwarp();
        if (e >= 0 && (peers & lt_mask) == 0) wcnt[warp][e] += __popc(peers);
        __syncwarp();
        ex[r] = e;
    }
    __syncthreads();
    for (int e = tid; e < E; e += kDispThreads) {
        int run = 0;
#pragma unroll
        for (int w = 0; w < kDispWarps; ++w) {
            const int c = wcnt[w][e];
            wcnt[w][e] = run;
            run += c;
        }
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < kRounds; ++r) {
        const int a = a_warp + r * 32 + lane;
        if (a >= A) continue;
        const int e = ex[r];
        int slot = -1;
        if (e >= 0) {
            const int g = base[size_t(blockIdx.x) * E + e] + wcnt[warp][e] + rank[r];
            if (g < off_s[e + 1] - off_s[e]) slot = off_s[e] + g;
        }
        slot_of[a] = slot;
        if (drop_mask != nullptr) drop_mask[a] = slot < 0 ? 1 : 0;
        if (slot >= 0) {
            perm[slot] = a;
            if (row_gate != nullptr) row_gate[slot] = gate[a];
        }
    }
}

// xp[row, :] = x[perm[row] / k, :] for row < offsets[E]; row_bytes % 16 == 0.
// With zero_out (top-1 direct output), also zero_out[t, :] = 0 for every token
// t whose assignment was dropped (slot_of[t] < 0).  Flattened over 16-byte
// pieces, eight independent loads in flight per thread.
__global__ void __launch_bounds__(256)
dispatch_gather_kernel(const uint8_t* __restrict__ x, int row_bytes, const int32_t* __restrict__ perm,
                       const int32_t* __restrict__ offsets, int E, int k, uint8_t* __restrict__ xp,
                       const int32_t* __restrict__ slot_of, int T, uint8_t* __restrict__ zero_out) {
    pdl_wait();
    pdl_release();
    const long long R = offsets[E];
    const int vecs = row_bytes >> 4;
    const long long copy_pieces = R * vecs;
    const long long pieces = copy_pieces + (zero_out != nullptr ? (long long)T * vecs : 0);
    const long long stride = (long long)gridDim.x * blockDim.x;
    constexpr int U = 8;
    for (long long p0 = (long long)blockIdx.x * blockDim.x + threadIdx.x; p0 < pieces; p0 += stride * U) {
        uint4 val[U];
        uint4* dst[U];
#pragma unroll
        for (int j = 0; j < U; ++j) {
            const long long pc = p0 + j * stride;
            dst[j] = nullptr;
            if (pc < copy_pieces) {
                const long long row = pc / vecs;
                const int v = int(pc - row * vecs);
                const int t = perm[row] / k;
                val[j] = __ldg(reinterpret_cast<const uint4*>(x + size_t(t) * row_bytes) + v);
                dst[j] = reinterpret_cast<uint4*>(xp) + pc;
            } else if (pc < pieces) {
                const long long q = pc - copy_pieces;
                const long long t = q / vecs;
                if (slot_of[t] < 0) {
                    val[j] = make_uint4(0u, 0u, 0u, 0u);
                    dst[j] = reinterpret_cast<uint4*>(zero_out) + q;
                }
            }
        }
#pragma unroll
        for (int j = 0; j < U; ++j)
            if (dst[j] != nullptr) *dst[j] = val[j];
    }
}

// ---------------------------------------------------------------------------
// Dispatch inside moe_forward.  The router already wrote, per chunk of
// chunk_tokens tokens (one router CTA), the expert histogram of its chunk
// and its per-expert probability sums; a chunk holds the chunk_tokens * k
// consecutive assignments of its tokens.
//   forward_scan_kernel     one CTA: bases, counts, capacity, offsets and
//                           the layer statistics
//   forward_permute_kernel  grid (chunks, G): stable in-chunk ranks, the
//                           dispatch arrays (y == 0 only), and the row
//                           gather split over the G CTAs of the chunk; for
//                           k == 1 with a direct output it also zero-fills the
//                           output rows of dropped tokens
// ---------------------------------------------------------------------------
constexpr int kFwdScanThreads = 1024;

// One CTA; warp w scans experts w, w+32, ...: 32 chunks per step, each lane
// one chunk, a warp prefix sum and a carried total (sums in fixed order).
__global__ void __launch_bounds__(kFwdScanThreads)
forward_scan_kernel(const int32_t* __restrict__ hist, const float* __restrict__ psum_part, int nchunk, int E,
                    int T, int k, int capacity, int32_t* __restrict__ base, int32_t* __restrict__ counts,
                    int32_t* __restrict__ offsets, moe_stats* __restrict__ st, int32_t* __restrict__ kept_out) {
    pdl_wait();
    pdl_release();
    __shared__ int kept[MOE_MAX_EXPERTS];
    __shared__ int cnt[MOE_MAX_EXPERTS];
    __shared__ float fp[MOE_MAX_EXPERTS];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int e = warp; e < E; e += kFwdScanThreads / 32) {
        int carry = 0;
        float ps = 0.f;
        for (int b0 = 0; b0 < nchunk; b0 += 32) {
            const int b = b0 + lane;
            const int h = b < nchunk ? hist[size_t(b) * E + e] : 0;
            if (psum_part != nullptr && b < nchunk) ps += psum_part[size_t(b) * E + e];
            int incl = h;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += v;
            }
            if (b < nchunk) base[size_t(b) * E + e] = carry + incl - h;
            carry += __shfl_sync(0xffffffffu, incl, 31);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
        if (lane == 0) {
            counts[e] = carry;
            cnt[e] = carry;
            kept[e] = capacity < 0 ? carry : min(carry, capacity);
            if (kept_out != nullptr) kept_out[e] = kept[e];
            fp[e] = (float(carry) / float(T)) * (ps / float(T));
        }
    }
    __syncthreads();
    if (threadIdx.x < 32) {
        constexpr int PER = MOE_MAX_EXPERTS / 32;
        int local[PER];
        int sum = 0;
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const int e = lane * PER + i;
            local[i] = e < E ? kept[e] : 0;
            sum += local[i];
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
            const int e = lane * PER + i;
            if (e < E) offsets[e] = run;
            run += local[i];
        }
        if (lane == 31) offsets[E] = incl;
        if (st != nullptr) {
            // statistics, in a fixed summation order
            float f = 0.f;
            int mx = 0;
#pragma unroll
            for (int i = 0; i < PER; ++i) {
                const int e = lane * PER + i;
                if (e < E) {
                    f += fp[e];
                    mx = max(mx, cnt[e]);
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                f += __shfl_xor_sync(0xffffffffu, f, o);
                mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            }
            if (lane == 31) {
                const int A = T * k;
                const int R = incl;
                st->aux_loss = float(E) * f;
                st->imbalance = float(mx) / (float(A) / float(E));
                st->drop_rate = float(A - R) / float(A);
                st->rows_kept = R;
                st->max_count = mx;
                st->dropped = A - R;
                st->rerouted = 0;
            }
        }
    }
}

constexpr int kFwdThreads = 256;
constexpr int kFwdMaxChunk = 1024;   // chunk_tokens * k
constexpr int kFwdRankRounds = kFwdMaxChunk / kDispWarps / 32;   // 4

// Stable ranks of a chunk's assignments within their expert (token order):
// warp w ranks the contiguous assignments [w*per, (w+1)*per) with peer
// masks, then wcnt[w][e] becomes the count of e in warps before w.  After
// the call, assignment i = w*per + r*32 + lane (in range) has expert ex[r]
// (-1 if outside [0,E)) and chunk rank wcnt[w][ex[r]] + rank[r].  All
// threads of the CTA call it; it ends with __syncthreads().
__device__ __forceinline__ int chunk_stable_ranks(const int32_t* __restrict__ idx, int a0, int na, int E,
                                                  int (*wcnt)[MOE_MAX_EXPERTS], int* ex, int* rank) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    for (int i = tid; i < kDispWarps * MOE_MAX_EXPERTS; i += kFwdThreads) (&wcnt[0][0])[i] = 0;
    __syncthreads();
    const int per = ((na + kDispWarps - 1) / kDispWarps + 31) & ~31;
    const uint32_t lt_mask = (1u << lane) - 1u;
#pragma unroll
    for (int r = 0; r < kFwdRankRounds; ++r) {
        const int i = warp * per + r * 32 + lane;
        const bool in = (r * 32 < per) && i < na;
        int e = in ? idx[a0 + i] : -1;
        if (e >= E || e < -1) e = -1;
        const uint32_t peers = __match_any_sync(0xffffffffu, e);
        const int local = __popc(peers & lt_mask);
        rank[r] = (e >= 0) ? wcnt[warp][e] + local : 0;
        __syncwarp();
        if (e >= 0 && (peers & lt_mask) == 0) wcnt[warp][e] += __popc(peers);
        __syncwarp();
        ex[r] = e;
    }
    __syncthreads();
    for (int e = tid; e < E; e += kFwdThreads) {
        int run = 0;
#pragma unroll
        for (int w = 0; w < kDispWarps; ++w) {
            const int c = wcnt[w][e];
            wcnt[w][e] = run;
            run += c;
        }
    }
    __syncthreads();
    return per;
}

// Gather of a chunk's grouped rows: xp[slot] = x[token] for every kept
// assignment (slot_s[i] >= 0, i = the assignment's index in the chunk), and,
// with out_zero_dropped, a zero output row for every token with no kept
// slot (k == 1 direct output).  The walk is over the chunk's tokens, not
// its assignments, so a token's row is read once and stored to each of its
// kept slots.  The chunk's tokens are split over the gridDim.y CTAs of the
// chunk (CTA y takes tokens y, y + Y, ...), flattened into 16-byte pieces
// with eight independent loads in flight per thread.  a0 and na are
// multiples of k (whole tokens).
__device__ __forceinline__ void gather_chunk_rows(const int* slot_s, int a0, int na, int k,
                                                  const uint8_t* __restrict__ x, int row_bytes,
                                                  uint8_t* __restrict__ xp, uint8_t* __restrict__ out_zero_dropped) {
    const int tid = threadIdx.x;
    const int vecs = row_bytes >> 4;
    const int Y = int(gridDim.y), y = int(blockIdx.y);
    const int t0 = a0 / k;
    const int nt = na / k;
    const int my_tokens = (nt - y + Y - 1) / Y;
    const int pieces = my_tokens * vecs;
    constexpr int U = 8;
    for (int p0 = tid; p0 < pieces; p0 += kFwdThreads * U) {
        uint4 val[U];
        int tl[U], vv[U], kind[U];   // kind 1: store to the token's kept slots, 2: zero its output row
        int first[U];                // the token's first slot (its only one for k = 1)
#pragma unroll
        for (int j = 0; j < U; ++j) {
            const int pc = p0 + j * kFwdThreads;
            kind[j] = 0;
            tl[j] = 0;
            vv[j] = 0;
            first[j] = -1;
            if (pc < pieces) {
                const int il = pc / vecs;
                vv[j] = pc - il * vecs;
                tl[j] = y + Y * il;
                first[j] = slot_s[tl[j] * k];
                bool kept = first[j] >= 0;
                for (int c = 1; c < k; ++c) kept |= slot_s[tl[j] * k + c] >= 0;
                if (kept) {
                    val[j] = __ldg(reinterpret_cast<const uint4*>(x + size_t(t0 + tl[j]) * row_bytes) + vv[j]);
                    kind[j] = 1;
                } else if (out_zero_dropped != nullptr) {
                    val[j] = make_uint4(0u, 0u, 0u, 0u);
                    kind[j] = 2;
                }
            }
        }
#pragma unroll
        for (int j = 0; j < U; ++j) {
            if (kind[j] == 1) {
                if (first[j] >= 0) reinterpret_cast<uint4*>(xp + size_t(first[j]) * row_bytes)[vv[j]] = val[j];
                for (int c = 1; c < k; ++c) {
                    const int slot = slot_s[tl[j] * k + c];
                    if (slot >= 0) reinterpret_cast<uint4*>(xp + size_t(slot) * row_bytes)[vv[j]] = val[j];
                }
            } else if (kind[j] == 2) {
                reinterpret_cast<uint4*>(out_zero_dropped + size_t(t0 + tl[j]) * row_bytes)[vv[j]] = val[j];
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Row gather by bulk copies (TMA, untiled cp.async.bulk; no multicast): one
// thread streams the CTA's token rows of x through a ring of shared-memory
// row buffers and stores each row to its kept slots of xp.  Addresses are
// 16-byte aligned and sizes multiples of 16 bytes (the host checks both).
// ---------------------------------------------------------------------------
constexpr int kGatherRing = 32;                  // at most this many row buffers
constexpr uint32_t kGatherSmem = 48u * 1024u;    // shared memory for the ring (and a zero row)
constexpr int kGatherLag = 2;                    // store groups in flight before a buffer is refilled
// Rows of fewer bytes use the thread-wide gather (ncu: bulk rows of 8 KB,
// large-top2: 50.0 -> 41.2 us; rows of 1.5-2 KB: 23 -> 31 us, 31 -> 34 us)
constexpr int kGatherBulkMinRow = 4096;

// global -> shared (this CTA), completion counted on `bar`
__device__ __forceinline__ void bulk_load_row(void* sdst, const void* gsrc, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(smem_u32(sdst)), "l"(reinterpret_cast<uint64_t>(gsrc)), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}
// shared -> global, in the thread's current bulk group
__device__ __forceinline__ void bulk_store_row(void* gdst, const void* ssrc, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;"
                 ::"l"(reinterpret_cast<uint64_t>(gdst)), "r"(smem_u32(ssrc)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// the source shared memory of all but the newest kGatherLag groups has been read
__device__ __forceinline__ void bulk_wait_read_lag() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(kGatherLag) : "memory");
}
// every bulk group of this thread has completed (its global writes done)
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Tokens of this CTA in a chunk: y, y + Y, ... below nt (Y = gridDim.y).
__device__ __forceinline__ int gather_my_tokens(int nt) {
    const int Y = int(gridDim.y), y = int(blockIdx.y);
    return (nt - y + Y - 1) / Y;
}

// Issued by one thread at the start: the first loads of the ring.
__device__ __forceinline__ void gather_tma_start(uint8_t* ring, int ring_rows, uint64_t* bars, int t0, int nt,
                                                 const uint8_t* __restrict__ x, int row_bytes) {
    const int Y = int(gridDim.y), y = int(blockIdx.y);
    const int my = gather_my_tokens(nt);
    for (int i = 0; i < ring_rows; ++i) mbar_init(&bars[i], 1);
    fence_barrier_init();
    for (int il = 0; il < min(ring_rows, my); ++il) {
        mbar_arrive_expect_tx(&bars[il], uint32_t(row_bytes));
        bulk_load_row(ring + size_t(il) * row_bytes, x + size_t(t0 + y + Y * il) * row_bytes, uint32_t(row_bytes),
                      &bars[il]);
    }
}

// Issued by the same thread once slot_s holds the chunk's slots: for each
// token, wait for its row, store it to each kept slot (or the zero row to
// its output row when every slot was dropped and out_zero_dropped is set),
// then refill the buffer of the token kGatherLag back with the row
// ring_rows ahead.  Ends when every store has completed.  A wait that gives
// up (2 s) records MOE_ERR_TIMEOUT; the loads already issued are still
// waited for before returning.
__device__ __forceinline__ void gather_tma_run(uint8_t* ring, int ring_rows, uint64_t* bars, const uint8_t* zero_row,
                                               const int* slot_s, int t0, int nt, int k,
                                               const uint8_t* __restrict__ x, int row_bytes,
                                               uint8_t* __restrict__ xp, uint8_t* __restrict__ out_zero_dropped,
                                               volatile int* abort_p) {
    const int Y = int(gridDim.y), y = int(blockIdx.y);
    const int my = gather_my_tokens(nt);
    int il = 0;
    for (; il < my; ++il) {
        const int b = il % ring_rows;
        if (!mbar_wait(&bars[b], uint32_t((il / ring_rows) & 1), abort_p)) break;
        const int tl = y + Y * il;
        const uint8_t* buf = ring + size_t(b) * row_bytes;
        bool any = false;
        for (int c = 0; c < k; ++c) {
            const int slot = slot_s[tl * k + c];
            if (slot >= 0) {
                bulk_store_row(xp + size_t(slot) * row_bytes, buf, uint32_t(row_bytes));
                any = true;
            }
        }
        if (!any && out_zero_dropped != nullptr)
            bulk_store_row(out_zero_dropped + size_t(t0 + tl) * row_bytes, zero_row, uint32_t(row_bytes));
        bulk_commit_group();
        const int nxt = il + ring_rows - kGatherLag;   // reuses the buffer of token il - kGatherLag
        if (il >= kGatherLag && nxt < my) {
            bulk_wait_read_lag();
            const int nb = nxt % ring_rows;
            mbar_arrive_expect_tx(&bars[nb], uint32_t(row_bytes));
            bulk_load_row(ring + size_t(nb) * row_bytes, x + size_t(t0 + y + Y * nxt) * row_bytes,
                          uint32_t(row_bytes), &bars[nb]);
        }
    }
    if (il < my) {
        // gave up: every load issued so far lands before the CTA may exit
        // loads went out for tokens [0, issued): the first ring_rows, then
        // one refill per iteration kGatherLag .. il-1
        const int issued = min(my, max(ring_rows, il + ring_rows - kGatherLag));
        for (int j = il; j < issued; ++j) mbar_wait_drain(&bars[j % ring_rows], uint32_t((j / ring_rows) & 1));
    }
    bulk_wait_all();
}

// drop_mask (nullable): 1 for dropped assignments, 0 for kept ones
__global__ void __launch_bounds__(kFwdThreads)
forward_permute_kernel(const int32_t* __restrict__ idx, const float* __restrict__ gate, int T, int k, int E,
                       int chunk_tokens, const int32_t* __restrict__ base, const int32_t* __restrict__ offsets,
                       int32_t* __restrict__ perm, int32_t* __restrict__ slot_of, float* __restrict__ row_gate,
                       const uint8_t* __restrict__ x, int row_bytes, uint8_t* __restrict__ xp,
                       uint8_t* __restrict__ out_zero_dropped, uint8_t* __restrict__ drop_mask) {
    pdl_wait();
    pdl_release();
    __shared__ int wcnt[kDispWarps][MOE_MAX_EXPERTS];
    __shared__ int off_s[MOE_MAX_EXPERTS + 1];
    __shared__ int slot_s[kFwdMaxChunk];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int chunk = blockIdx.x;
    const int A = T * k;
    const int a0 = chunk * chunk_tokens * k;
    const int na = min(chunk_tokens * k, A - a0);
    for (int e = tid; e <= E; e += kFwdThreads) off_s[e] = offsets[e];
    int ex[kFwdRankRounds], rank[kFwdRankRounds];
    const int per = chunk_stable_ranks(idx, a0, na, E, wcnt, ex, rank);
    const bool writer = blockIdx.y == 0;
#pragma unroll
    for (int r = 0; r < kFwdRankRounds; ++r) {
        const int i = warp * per + r * 32 + lane;
        if (!((r * 32 < per) && i < na)) continue;
        const int a = a0 + i;
        const int e = ex[r];
        int slot = -1;
        if (e >= 0) {
            const int g = base[size_t(chunk) * E + e] + wcnt[warp][e] + rank[r];
            if (g < off_s[e + 1] - off_s[e]) slot = off_s[e] + g;
        }
        slot_s[i] = slot;
        if (writer) {
            slot_of[a] = slot;
            if (drop_mask != nullptr) drop_mask[a] = slot < 0 ? 1 : 0;
            if (slot >= 0) {
                perm[slot] = a;
                if (row_gate != nullptr) row_gate[slot] = gate[a];
            }
        }
    }
    __syncthreads();
    gather_chunk_rows(slot_s, a0, na, k, x, row_bytes, xp, out_zero_dropped);
}

// The scan fused into the permute: every CTA of chunk c derives what the
// one-CTA scan would give it from the router's per-chunk histograms (its
// bases: counts of each expert in chunks before c; the totals, capacity
// clamp and offsets), so the dispatch is one launch.  CTA (0, 0) also
// writes counts, offsets and the statistics.  Each CTA reads nchunk * E
// histogram entries, so the host uses this only while that table is small.
// Thread e < E owns expert e (E <= MOE_MAX_EXPERTS = kFwdThreads).
static_assert(MOE_MAX_EXPERTS <= kFwdThreads, "one thread per expert");

__global__ void __launch_bounds__(kFwdThreads)
forward_dispatch_kernel(const int32_t* __restrict__ idx, const float* __restrict__ gate, int T, int k, int E,
                        int chunk_tokens, const int32_t* __restrict__ hist, const float* __restrict__ psum_part,
                        int nchunk, int capacity, int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                        moe_stats* __restrict__ st, int32_t* __restrict__ perm, int32_t* __restrict__ slot_of,
                        float* __restrict__ row_gate, const uint8_t* __restrict__ x, int row_bytes,
                        uint8_t* __restrict__ xp, uint8_t* __restrict__ out_zero_dropped, int ring_rows) {
    pdl_wait();
    pdl_release();
    // ring_rows > 0: the row gather runs on bulk copies through ring_rows
    // row buffers in dynamic shared memory (then a zero row, for
    // out_zero_dropped); its first loads go out now, under the scan
    extern __shared__ __align__(128) uint8_t g_ring[];
    __shared__ __align__(8) uint64_t g_bar[kGatherRing];
    __shared__ int g_abort;
    if (ring_rows > 0) {
        if (threadIdx.x == 0) {
            g_abort = 0;
            gather_tma_start(g_ring, ring_rows, g_bar, blockIdx.x * chunk_tokens,
                             min(chunk_tokens, T - int(blockIdx.x) * chunk_tokens), x, row_bytes);
        }
        if (out_zero_dropped != nullptr) {
            uint4* z = reinterpret_cast<uint4*>(g_ring + size_t(ring_rows) * row_bytes);
            for (int i = threadIdx.x; i < (row_bytes >> 4); i += kFwdThreads) z[i] = make_uint4(0u, 0u, 0u, 0u);
            fence_proxy_async_smem();   // the bulk stores (async proxy) read these zeros
        }
    }
    __shared__ int wcnt[kDispWarps][MOE_MAX_EXPERTS];
    __shared__ int off_s[MOE_MAX_EXPERTS + 1];
    __shared__ int base_s[MOE_MAX_EXPERTS];
    __shared__ int kept_s[MOE_MAX_EXPERTS];
    __shared__ int cnt_s[MOE_MAX_EXPERTS];
    __shared__ float fp_s[MOE_MAX_EXPERTS];
    __shared__ int slot_s[kFwdMaxChunk];
    __shared__ int red_pre[kFwdThreads], red_tot[kFwdThreads];
    __shared__ float red_ps[kFwdThreads];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int chunk = blockIdx.x;
    const bool lead = (blockIdx.x == 0 && blockIdx.y == 0);
    const int A = T * k;
    const int a0 = chunk * chunk_tokens * k;
    const int na = min(chunk_tokens * k, A - a0);

    // Per-expert totals and this chunk's bases from the router's per-chunk
    // histograms.  The whole CTA sums: thread (part, e) takes chunks part,
    // part + parts, ... of expert e (loads coalesced across experts), then
    // thread e adds the parts' partial sums in part order (a fixed order:
    // the probability sums are reproducible run to run).  The loop is
    // unrolled 16 deep so that a thread's table loads (32 at E = 64 and
    // 128 tiles) go out together rather than a few per L2 round trip.
    const int parts = kFwdThreads / E;   // >= 1
    if (tid < parts * E) {
        const int e = tid % E, part = tid / E;
        int pre = 0, tot = 0;
        float ps = 0.f;
#pragma unroll 16
        for (int b = part; b < nchunk; b += parts) {
            const int h = hist[size_t(b) * E + e];
            tot += h;
            pre += (b < chunk) ? h : 0;
        }
        if (lead && st != nullptr && psum_part != nullptr)
            for (int b = part; b < nchunk; b += parts) ps += psum_part[size_t(b) * E + e];
        red_pre[tid] = pre;
        red_tot[tid] = tot;
        red_ps[tid] = ps;
    }
    __syncthreads();
    if (tid < E) {
        const int e = tid;
        int pre = 0, tot = 0;
        float ps = 0.f;
        for (int p = 0; p < parts; ++p) {
            pre += red_pre[p * E + e];
            tot += red_tot[p * E + e];
            ps += red_ps[p * E + e];
        }
        base_s[e] = pre;
        cnt_s[e] = tot;
        kept_s[e] = capacity < 0 ? tot : min(tot, capacity);
        fp_s[e] = (float(tot) / float(T)) * (ps / float(T));
        if (lead) counts[e] = tot;
    }
    __syncthreads();
    if (warp == 0) {
        constexpr int PER = MOE_MAX_EXPERTS / 32;
        int local[PER];
        int sum = 0;
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const int e = lane * PER + i;
            local[i] = e < E ? kept_s[e] : 0;
            sum += local[i];
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
            const int e = lane * PER + i;
            if (e < E) off_s[e] = run;
            run += local[i];
        }
        if (lane == 31) off_s[E] = incl;
        if (lead && st != nullptr) {
            // statistics, in a fixed summation order
            float f = 0.f;
            int mx = 0;
#pragma unroll
            for (int i = 0; i < PER; ++i) {
                const int e = lane * PER + i;
                if (e < E) {
                    f += fp_s[e];
                    mx = max(mx, cnt_s[e]);
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                f += __shfl_xor_sync(0xffffffffu, f, o);
                mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            }
            if (lane == 31) {
                const int R = incl;
                st->aux_loss = float(E) * f;
                st->imbalance = float(mx) / (float(A) / float(E));
                st->drop_rate = float(A - R) / float(A);
                st->rows_kept = R;
                st->max_count = mx;
                st->dropped = A - R;
                st->rerouted = 0;
            }
        }
    }
    __syncthreads();
    if (lead)
        for (int e = tid; e <= E; e += kFwdThreads) offsets[e] = off_s[e];

    int ex[kFwdRankRounds], rank[kFwdRankRounds];
    const int per = chunk_stable_ranks(idx, a0, na, E, wcnt, ex, rank);
    const bool writer = blockIdx.y == 0;
#pragma unroll
    for (int r = 0; r < kFwdRankRounds; ++r) {
        const int i = warp * per + r * 32 + lane;
        if (!((r * 32 < per) && i < na)) continue;
        const int a = a0 + i;
        const int e = ex[r];
        int slot = -1;
        if (e >= 0) {
            const int g = base_s[e] + wcnt[warp][e] + rank[r];
            if (g < off_s[e + 1] - off_s[e]) slot = off_s[e] + g;
        }
        slot_s[i] = slot;
        if (writer) {
            slot_of[a] = slot;
            if (slot >= 0) {
                perm[slot] = a;
                if (row_gate != nullptr) row_gate[slot] = gate[a];
            }
        }
    }
    __syncthreads();
    if (ring_rows > 0) {
        if (threadIdx.x == 0)
            gather_tma_run(g_ring, ring_rows, g_bar, g_ring + size_t(ring_rows) * row_bytes, slot_s,
                           int(blockIdx.x) * chunk_tokens, na / k, k, x, row_bytes, xp, out_zero_dropped, &g_abort);
    } else {
        gather_chunk_rows(slot_s, a0, na, k, x, row_bytes, xp, out_zero_dropped);
    }
}

// ---------------------------------------------------------------------------
// Overflow rerouting (F rounds).  Round r = 1..F: every token with an
// unserved slot offers its first unserved slot j to its r-th fallback
// expert c = fb_idx[t, r-1]; c accepts offers in token order while it holds
// fewer than `capacity` rows.  Expert e's rows: its own kept assignments
// (token order), then round 1's accepted offers (token order), round 2's...
//
// Per-assignment state: srv[a] = 0 kept by its own expert, r >= 1 served in
// round r, -1 not served (yet); srank[a] = its rank among the rows its
// expert took in that round.  Per token: otok[t] = slot offered in the
// current round (-1: none), orank[t] = the offer's rank among the chunk's
// offers to the same expert.
//
//   reroute_mark_kernel(r)   grid (chunks): round 1 first ranks the chunk's
//                            own assignments (srv / srank); round r > 1
//                            first settles round r-1's offers; then it
//                            makes round r's offers and their per-chunk
//                            histogram
//   reroute_scan_kernel(r)   one CTA: per-(chunk, expert) bases of round r's
//                            offers, how many each expert accepts, the
//                            experts' loads; after round F the final
//                            offsets and statistics
//   reroute_permute_kernel   grid (chunks, G): settles round F's offers,
//                            writes the dispatch arrays and gathers rows
// ---------------------------------------------------------------------------
// Step-level input of a rerouting dispatch: splits ranked [T, k+F] (each
// token's experts in router order) into its own choices idx/gate [T, k]
// and fallbacks fb_idx/fb_gate [T, F], and writes each chunk's histogram of
// the own choices.  An own choice outside [0, E) is counted nowhere (it is
// dropped) and raises MOE_ERR_BAD_ROUTING; a fallback outside [0, E) is
// never offered.  ranked_gate may be null (gates then read as 0).
__global__ void __launch_bounds__(kFwdThreads)
reroute_split_kernel(const int32_t* __restrict__ ranked_idx, const float* __restrict__ ranked_gate, int T, int k,
                     int F, int E, int chunk_tokens, int32_t* __restrict__ idx, float* __restrict__ gate,
                     int32_t* __restrict__ fb_idx, float* __restrict__ fb_gate, int32_t* __restrict__ hist) {
    pdl_wait();
    pdl_release();
    __shared__ int h[MOE_MAX_EXPERTS];
    for (int e = threadIdx.x; e < E; e += kFwdThreads) h[e] = 0;
    __syncthreads();
    const int K = k + F;
    const int t0 = blockIdx.x * chunk_tokens;
    const int nt = min(chunk_tokens, T - t0);
    for (int i = threadIdx.x; i < nt * K; i += kFwdThreads) {
        const int t = t0 + i / K;
        const int c = i - (i / K) * K;
        const int v = ranked_idx[size_t(t) * K + c];
        const float g = ranked_gate != nullptr ? ranked_gate[size_t(t) * K + c] : 0.f;
        if (c < k) {
            idx[size_t(t) * k + c] = v;
            gate[size_t(t) * k + c] = g;
            if (v >= 0 && v < E)
                atomicAdd(&h[v], 1);
            else
                set_error(MOE_ERR_BAD_ROUTING);
        } else {
            fb_idx[size_t(t) * F + (c - k)] = v;
            fb_gate[size_t(t) * F + (c - k)] = g;
        }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += kFwdThreads) hist[size_t(blockIdx.x) * E + e] = h[e];
}

__global__ void __launch_bounds__(kFwdThreads)
reroute_mark_kernel(const int32_t* __restrict__ idx, int T, int k, int E, int chunk_tokens, int capacity,
                    const int32_t* __restrict__ base, const int32_t* __restrict__ fb_idx, int F, int r,
                    const int32_t* __restrict__ prev_rbase, const int32_t* __restrict__ prev_acc,
                    int32_t* __restrict__ srv, int32_t* __restrict__ srank, int32_t* __restrict__ otok,
                    int32_t* __restrict__ orank, int32_t* __restrict__ rhist) {
    pdl_wait();
    pdl_release();
    __shared__ int wcnt[kDispWarps][MOE_MAX_EXPERTS];
    __shared__ int srv_s[kFwdMaxChunk];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int chunk = blockIdx.x;
    const int t0 = chunk * chunk_tokens;
    const int nt = min(chunk_tokens, T - t0);
    const int a0 = t0 * k;
    const int na = nt * k;
    if (r == 1) {
        int ex[kFwdRankRounds], rank[kFwdRankRounds];
        const int per = chunk_stable_ranks(idx, a0, na, E, wcnt, ex, rank);
#pragma unroll
        for (int q = 0; q < kFwdRankRounds; ++q) {
            const int i = warp * per + q * 32 + lane;
            if (!((q * 32 < per) && i < na)) continue;
            const int e = ex[q];
            int sv = -1, g = 0;
            if (e >= 0) {
                g = base[size_t(chunk) * E + e] + wcnt[warp][e] + rank[q];
                if (g < capacity) sv = 0;
            }
            srv_s[i] = sv;
            srv[a0 + i] = sv;
            srank[a0 + i] = g;
        }
    } else {
        for (int i = tid; i < na; i += kFwdThreads) srv_s[i] = srv[a0 + i];
        __syncthreads();
        // settle round r-1: an offer is accepted when its rank among all
        // offers to its expert is below what that expert accepted
        for (int i = tid; i < nt; i += kFwdThreads) {
            const int t = t0 + i;
            const int j = otok[t];
            if (j < 0) continue;
            const int c = fb_idx[size_t(t) * F + (r - 2)];
            const int g = prev_rbase[size_t(chunk) * E + c] + orank[t];
            if (g < prev_acc[c]) {
                srv_s[i * k + j] = r - 1;
                srv[a0 + i * k + j] = r - 1;
                srank[a0 + i * k + j] = g;
            }
        }
    }
    __syncthreads();   // every read of wcnt above is done; srv_s is complete
    for (int i = tid; i < kDispWarps * MOE_MAX_EXPERTS; i += kFwdThreads) (&wcnt[0][0])[i] = 0;
    __syncthreads();
    // round r's offers: token i of the chunk is thread i (chunk_tokens <= 128)
    const uint32_t lt_mask = (1u << lane) - 1u;
    int c = -1, j = -1, local = 0;
    if (tid < nt) {
        for (int jj = 0; jj < k; ++jj)
            if (srv_s[tid * k + jj] < 0) {
                j = jj;
                break;
            }
        if (j >= 0) c = fb_idx[size_t(t0 + tid) * F + (r - 1)];
        if (c >= E || c < 0) {   // a fallback outside [0, E) cannot be served
            c = -1;
            j = -1;
        }
    }
    if (tid < 128) {
        const uint32_t peers = __match_any_sync(0xffffffffu, c);
        local = __popc(peers & lt_mask);
        if (c >= 0 && (peers & lt_mask) == 0) wcnt[warp][c] = __popc(peers);
    }
    __syncthreads();
    if (tid < nt) {
        int before = 0;
        if (c >= 0)
            for (int w = 0; w < warp; ++w) before += wcnt[w][c];
        otok[t0 + tid] = j;
        orank[t0 + tid] = before + local;
    }
    for (int e = tid; e < E; e += kFwdThreads) {
        int tot = 0;
#pragma unroll
        for (int w = 0; w < 4; ++w) tot += wcnt[w][e];
        rhist[size_t(chunk) * E + e] = tot;
    }
}

// One CTA; warp w scans experts w, w+32, ... over the chunks (fixed order).
// load [E]: rows each expert holds (in: before round r, out: after).
__global__ void __launch_bounds__(kFwdScanThreads)
reroute_scan_kernel(const int32_t* __restrict__ rhist, int nchunk, int E, int capacity, int r, int F, int T, int k,
                    int32_t* __restrict__ rbase, int32_t* __restrict__ load, int32_t* __restrict__ acc,
                    int32_t* __restrict__ start, int32_t* __restrict__ offsets, moe_stats* __restrict__ st) {
    pdl_wait();
    pdl_release();
    __shared__ int load_s[MOE_MAX_EXPERTS];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int e = warp; e < E; e += kFwdScanThreads / 32) {
        int carry = 0;
        for (int b0 = 0; b0 < nchunk; b0 += 32) {
            const int b = b0 + lane;
            const int h = b < nchunk ? rhist[size_t(b) * E + e] : 0;
            int incl = h;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += v;
            }
            if (b < nchunk) rbase[size_t(b) * E + e] = carry + incl - h;
            carry += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) {
            const int l = load[e];
            const int a = min(carry, max(capacity - l, 0));
            acc[e] = a;
            start[e] = l;
            load[e] = l + a;
            load_s[e] = l + a;
        }
    }
    if (r != F) return;
    __syncthreads();
    if (threadIdx.x < 32) {
        constexpr int PER = MOE_MAX_EXPERTS / 32;
        int local[PER];
        int sum = 0;
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const int e = lane * PER + i;
            local[i] = e < E ? load_s[e] : 0;
            sum += local[i];
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
            const int e = lane * PER + i;
            if (e < E) offsets[e] = run;
            run += local[i];
        }
        if (lane == 31) {
            offsets[E] = incl;
            if (st != nullptr) {
                // the primary dispatch's statistics are already in st
                const int A = T * k;
                const int R = incl;
                st->rerouted = R - st->rows_kept;
                st->rows_kept = R;
                st->dropped = A - R;
                st->drop_rate = float(A - R) / float(A);
            }
        }
    }
}

// start: [F][E] row start of each round's accepted offers within an expert
__global__ void __launch_bounds__(kFwdThreads)
reroute_permute_kernel(const int32_t* __restrict__ idx, const float* __restrict__ gate,
                       const int32_t* __restrict__ fb_idx, const float* __restrict__ fb_gate, int T, int k, int E,
                       int F, int chunk_tokens, const int32_t* __restrict__ srv, const int32_t* __restrict__ srank,
                       const int32_t* __restrict__ otok, const int32_t* __restrict__ orank,
                       const int32_t* __restrict__ last_rbase, const int32_t* __restrict__ last_acc,
                       const int32_t* __restrict__ start, const int32_t* __restrict__ offsets,
                       int32_t* __restrict__ perm, int32_t* __restrict__ slot_of, float* __restrict__ row_gate,
                       const uint8_t* __restrict__ x, int row_bytes, uint8_t* __restrict__ xp,
                       uint8_t* __restrict__ out_zero_dropped, uint8_t* __restrict__ drop_mask) {
    pdl_wait();
    pdl_release();
    __shared__ int off_s[MOE_MAX_EXPERTS + 1];
    __shared__ int slot_s[kFwdMaxChunk];
    const int tid = threadIdx.x;
    const int chunk = blockIdx.x;
    const int t0 = chunk * chunk_tokens;
    const int nt = min(chunk_tokens, T - t0);
    const int a0 = t0 * k;
    const int na = nt * k;
    for (int e = tid; e <= E; e += kFwdThreads) off_s[e] = offsets[e];
    __syncthreads();
    const bool writer = blockIdx.y == 0;
    for (int i = tid; i < na; i += kFwdThreads) {
        const int a = a0 + i;
        const int t = a / k;
        const int j = a - t * k;
        const int sv = srv[a];
        int slot = -1;
        float g = 0.f;
        if (sv == 0) {
            const int e = idx[a];
            slot = off_s[e] + srank[a];
            g = gate[a];
        } else if (sv > 0) {
            const int c = fb_idx[size_t(t) * F + (sv - 1)];
            slot = off_s[c] + start[size_t(sv - 1) * E + c] + srank[a];
            g = fb_gate[size_t(t) * F + (sv - 1)];
        } else if (otok[t] == j) {
            const int c = fb_idx[size_t(t) * F + (F - 1)];
            const int gg = last_rbase[size_t(chunk) * E + c] + orank[t];
            if (gg < last_acc[c]) {
                slot = off_s[c] + start[size_t(F - 1) * E + c] + gg;
                g = fb_gate[size_t(t) * F + (F - 1)];
            }
        }
        slot_s[i] = slot;
        if (writer) {
            slot_of[a] = slot;
            if (drop_mask != nullptr) drop_mask[a] = slot < 0 ? 1 : 0;
            if (slot >= 0) {
                perm[slot] = a;
                if (row_gate != nullptr) row_gate[slot] = g;
            }
        }
    }
    __syncthreads();
    gather_chunk_rows(slot_s, a0, na, k, x, row_bytes, xp, out_zero_dropped);
}

// ---------------------------------------------------------------------------
// Step 4: combine.  out[t] = sum over kept slots j (in slot order) of
// w_tj * yp[slot_of[t*k+j]]; w_tj = gate or 1.  fp32 accumulation.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void load8(const float* p, float (&v)[8]) {
    const float4 a = *reinterpret_cast<const float4*>(p);
    const float4 b = *reinterpret_cast<const float4*>(p + 4);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float (&v)[8]) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    v[0] = bf16_lo(u.x); v[1] = bf16_hi(u.x); v[2] = bf16_lo(u.y); v[3] = bf16_hi(u.y);
    v[4] = bf16_lo(u.z); v[5] = bf16_hi(u.z); v[6] = bf16_lo(u.w); v[7] = bf16_hi(u.w);
}
__device__ __forceinline__ void store8(float* p, const float (&v)[8]) {
    *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
    *reinterpret_cast<float4*>(p + 4) = make_float4(v[4], v[5], v[6], v[7]);
}
__device__ __forceinline__ void store8(__nv_bfloat16* p, const float (&v)[8]) {
    uint4 u;
    u.x = pack_bf16x2(v[0], v[1]); u.y = pack_bf16x2(v[2], v[3]);
    u.z = pack_bf16x2(v[4], v[5]); u.w = pack_bf16x2(v[6], v[7]);
    *reinterpret_cast<uint4*>(p) = u;
}

// One warp per token, the warps striding over the tokens (the grid is what
// fits on the GPU at once); each lane handles 16-byte pieces of the row,
// four at a time, so 4 * k independent loads are in flight before the adds.
// Lane j < k holds slot j's row and gate, loaded one token ahead so the
// next token's indices arrive while this token's rows load.  With S > 0
// shared experts, ys [S, Tn, d] holds their outputs and each adds its row
// of token t with weight 1 after the routed slots.
template <typename T>
__global__ void __launch_bounds__(256)
combine_kernel(const T* __restrict__ yp, const int32_t* __restrict__ slot_of, const float* __restrict__ gate,
               int Tn, int k, int d, T* __restrict__ out, const T* __restrict__ ys, int S) {
    pdl_wait();
    pdl_release();
    constexpr int EPV = 16 / sizeof(T);   // elements per 16-byte piece
    constexpr int U = 4;
    const int warps_total = gridDim.x * (blockDim.x >> 5);
    const int lane = threadIdx.x & 31;
    const int pieces = d / EPV;
    auto fetch = [&](int tt, int& sl, float& wv) {
        sl = -1;
        wv = 1.f;
        if (tt < Tn && lane < k) {
            sl = slot_of[size_t(tt) * k + lane];
            if (gate != nullptr) wv = gate[size_t(tt) * k + lane];
        }
    };
    int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    int next_slot;
    float next_w;
    fetch(t, next_slot, next_w);
    for (; t < Tn; t += warps_total) {
        int slot[MOE_MAX_TOPK];
        float w[MOE_MAX_TOPK];
#pragma unroll
        for (int j = 0; j < MOE_MAX_TOPK; ++j) {
            slot[j] = __shfl_sync(0xffffffffu, next_slot, j);
            w[j] = __shfl_sync(0xffffffffu, next_w, j);
        }
        fetch(t + warps_total, next_slot, next_w);
        for (int c0 = lane; c0 < pieces; c0 += 32 * U) {
            float acc[U][EPV];
#pragma unroll
            for (int u = 0; u < U; ++u)
#pragma unroll
                for (int i = 0; i < EPV; ++i) acc[u][i] = 0.f;
            // routed slots (the unrolled loop lets all k rows' loads be in
            // flight together), then the shared experts' rows one at a time
            auto add_row = [&](const T* src, float wj) {
                uint4 raw[U];
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int c = c0 + u * 32;
                    raw[u] = (c < pieces) ? __ldg(reinterpret_cast<const uint4*>(src) + c)
                                          : make_uint4(0u, 0u, 0u, 0u);
                }
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    float v[8];
                    if constexpr (sizeof(T) == 2) {
                        v[0] = bf16_lo(raw[u].x); v[1] = bf16_hi(raw[u].x); v[2] = bf16_lo(raw[u].y);
                        v[3] = bf16_hi(raw[u].y); v[4] = bf16_lo(raw[u].z); v[5] = bf16_hi(raw[u].z);
                        v[6] = bf16_lo(raw[u].w); v[7] = bf16_hi(raw[u].w);
                    } else {
                        v[0] = __uint_as_float(raw[u].x); v[1] = __uint_as_float(raw[u].y);
                        v[2] = __uint_as_float(raw[u].z); v[3] = __uint_as_float(raw[u].w);
                    }
#pragma unroll
                    for (int i = 0; i < EPV; ++i) acc[u][i] = fmaf(wj, v[i], acc[u][i]);
                }
            };
#pragma unroll
            for (int j = 0; j < MOE_MAX_TOPK; ++j)
                if (slot[j] >= 0) add_row(yp + size_t(slot[j]) * d, w[j]);
#pragma unroll 1
            for (int sx = 0; sx < S; ++sx) add_row(ys + (size_t(sx) * Tn + t) * d, 1.f);
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int c = c0 + u * 32;
                if (c >= pieces) continue;
                uint4 o;
                if constexpr (sizeof(T) == 2) {
                    o.x = pack_bf16x2(acc[u][0], acc[u][1]);
                    o.y = pack_bf16x2(acc[u][2], acc[u][3]);
                    o.z = pack_bf16x2(acc[u][4], acc[u][5]);
                    o.w = pack_bf16x2(acc[u][6], acc[u][7]);
                } else {
                    o = make_uint4(__float_as_uint(acc[u][0]), __float_as_uint(acc[u][1]),
                                   __float_as_uint(acc[u][2]), __float_as_uint(acc[u][3]));
                }
                reinterpret_cast<uint4*>(out + size_t(t) * d)[c] = o;
            }
        }
    }
}

// Exercises the bounded-wait path: waits on an mbarrier that nothing ever
// completes, gives up after limit_ns and records MOE_ERR_TIMEOUT, like a
// pipeline wait of the layer's kernels that runs out.
__global__ void wait_timeout_probe_kernel(uint64_t limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, limit_ns);
    __syncthreads();
}

// y[i] = GELU(x[i]) with the form the fp32 path uses (variant 0, erff) or the
// bf16 tensor-core epilogue uses (variant 1, A&S 7.1.26); for testing.
__global__ void gelu_probe_kernel(const float* __restrict__ x, float* __restrict__ y, int n, int variant) {
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x)
        y[i] = variant == 0 ? gelu_erf(x[i]) : gelu_as(x[i]);
}

// ---------------------------------------------------------------------------
// statistics (one CTA)
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
stats_kernel(const int32_t* __restrict__ counts, const int32_t* __restrict__ offsets,
             const float* __restrict__ prob_sum, int T, int k, int E, moe_stats* __restrict__ st) {
    pdl_wait();
    pdl_release();
    __shared__ float s_fp[256];
    __shared__ int s_max[256];
    float fp = 0.f;
    int mx = 0;
    const float invT = 1.0f / float(T);
    for (int e = threadIdx.x; e < E; e += 256) {
        fp += (float(counts[e]) * invT) * (prob_sum[e] * invT);
        mx = max(mx, counts[e]);
    }
    s_fp[threadIdx.x] = fp;
    s_max[threadIdx.x] = mx;
    __syncthreads();
    for (int o = 128; o > 0; o >>= 1) {
        if (threadIdx.x < o) {
            s_fp[threadIdx.x] += s_fp[threadIdx.x + o];
            s_max[threadIdx.x] = max(s_max[threadIdx.x], s_max[threadIdx.x + o]);
        }
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        const int A = T * k;
        const int R = offsets[E];
        st->aux_loss = float(E) * s_fp[0];
        st->imbalance = float(s_max[0]) / (float(A) / float(E));
        st->drop_rate = float(A - R) / float(A);
        st->rows_kept = R;
        st->max_count = s_max[0];
        st->dropped = A - R;
        st->rerouted = 0;
    }
}

}  // namespace moe
