// libmoe: host side of the C ABI declared in include/moe.h.
//
// Every entry point validates its arguments before touching the GPU, then
// enqueues kernels on the caller's stream.  Nothing here synchronises the
// host except moe_get_error, moe_timing_read and the pipeline's run and
// destroy, and nothing allocates device memory: scratch comes from the
// caller's workspace.  The pipeline (pipeline.cuh) owns only streams,
// events and graphs.
#include <algorithm>
#include <atomic>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "common.cuh"
#include "dispatch.cuh"
#include "ffn.cuh"
#include "ffn_f32.cuh"
#include "router.cuh"

using namespace moe;

namespace {

// ---------------------------------------------------------------------------
// NVTX ranges: one around every entry point that enqueues work and one
// around every kernel launch, so that a profiler timeline (Nsight Systems,
// or torch.profiler recording NVTX) shows the router, the dispatch, the two
// FFN GEMMs and the combine apart.  Off unless the environment variable
// MOE_NVTX is "1" when the library first checks, or moe_trace_enable(1) is
// called; off, a range costs one relaxed atomic load.
// ---------------------------------------------------------------------------
std::atomic<int> g_trace{-1};

bool trace_on() {
    int v = g_trace.load(std::memory_order_relaxed);
    if (v < 0) {
        const char* e = std::getenv("MOE_NVTX");
        int want = (e != nullptr && e[0] == '1') ? 1 : 0;
        int expected = -1;
        g_trace.compare_exchange_strong(expected, want, std::memory_order_relaxed);
        v = g_trace.load(std::memory_order_relaxed);
    }
    return v == 1;
}

class TraceRange {
  public:
    explicit TraceRange(const char* name) : on_(trace_on()) {
        if (on_) nvtxRangePushA(name);
    }
    ~TraceRange() {
        if (on_) nvtxRangePop();
    }
    TraceRange(const TraceRange&) = delete;
    TraceRange& operator=(const TraceRange&) = delete;

  private:
    bool on_;
};

const char* kernel_range_name(int kernel) {
    static const char* const names[MOE_NUM_KERNELS] = {
        "moe.kernel.router", "moe.kernel.count", "moe.kernel.scan", "moe.kernel.permute", "moe.kernel.gather",
        "moe.kernel.ffn1",   "moe.kernel.ffn2",  "moe.kernel.combine", "moe.kernel.stats", "moe.kernel.reroute"};
    return (kernel >= 0 && kernel < MOE_NUM_KERNELS && names[kernel]) ? names[kernel] : "moe.kernel";
}

// ---------------------------------------------------------------------------
// launch counter and optional per-kernel event timing
// ---------------------------------------------------------------------------
std::atomic<uint64_t> g_launches{0};

struct TimedLaunch {
    int kernel;
    cudaEvent_t start, stop;
};

struct TimingState {
    std::mutex mu;
    bool enabled = false;
    std::vector<cudaEvent_t> free_events;
    std::vector<TimedLaunch> pending;
    double ms[MOE_NUM_KERNELS] = {};
    int64_t launches[MOE_NUM_KERNELS] = {};
};
TimingState g_timing;

constexpr int kEventPool = 4096;

// caller holds g_timing.mu
void harvest_locked(size_t upto) {
    for (size_t i = 0; i < upto && i < g_timing.pending.size(); ++i) {
        TimedLaunch& t = g_timing.pending[i];
        float ms = 0.f;
        if (cudaEventSynchronize(t.stop) == cudaSuccess && cudaEventElapsedTime(&ms, t.start, t.stop) == cudaSuccess) {
            g_timing.ms[t.kernel] += ms;
            g_timing.launches[t.kernel] += 1;
        }
        g_timing.free_events.push_back(t.start);
        g_timing.free_events.push_back(t.stop);
    }
    g_timing.pending.erase(g_timing.pending.begin(),
                           g_timing.pending.begin() + std::min(upto, g_timing.pending.size()));
}

cudaEvent_t take_event_locked() {
    if (g_timing.free_events.empty()) harvest_locked(g_timing.pending.size() / 2 + 1);
    if (g_timing.free_events.empty()) return nullptr;
    cudaEvent_t e = g_timing.free_events.back();
    g_timing.free_events.pop_back();
    return e;
}

// Brackets one kernel launch: records the start event (when timing is on)
// and, in finish(), checks the launch, counts it and records the stop event.
class Launch {
  public:
    Launch(int kernel, cudaStream_t s) : trace_(kernel_range_name(kernel)), kernel_(kernel), stream_(s) {
        if (g_timing.enabled) {
            std::lock_guard<std::mutex> lk(g_timing.mu);
            start_ = take_event_locked();
            if (start_ != nullptr) cudaEventRecord(start_, stream_);
        }
    }
    int finish(cudaError_t launch_err = cudaSuccess) {
        const cudaError_t last = cudaGetLastError();
        const cudaError_t err = launch_err != cudaSuccess ? launch_err : last;
        g_launches.fetch_add(1, std::memory_order_relaxed);
        if (start_ != nullptr) {
            std::lock_guard<std::mutex> lk(g_timing.mu);
            cudaEvent_t stop = take_event_locked();
            if (stop != nullptr) {
                cudaEventRecord(stop, stream_);
                g_timing.pending.push_back({kernel_, start_, stop});
            } else {
                g_timing.free_events.push_back(start_);
            }
        }
        if (err != cudaSuccess) {
            std::fprintf(stderr, "libmoe: kernel %d launch failed: %s\n", kernel_, cudaGetErrorString(err));
            return MOE_ERR_CUDA;
        }
        return MOE_OK;
    }

  private:
    TraceRange trace_;
    int kernel_;
    cudaStream_t stream_;
    cudaEvent_t start_ = nullptr;
};

// Every kernel of the library asks for the largest shared-memory carveout,
// so consecutive kernels of a step never reconfigure an SM's L1/shared
// split between them (set once per kernel and device).
std::mutex g_carve_mu;
std::vector<std::pair<const void*, int>> g_carve_done;

inline void uniform_carveout(const void* kern) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return;
    std::lock_guard<std::mutex> lk(g_carve_mu);
    for (const auto& kd : g_carve_done)
        if (kd.first == kern && kd.second == dev) return;
    cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, int(cudaSharedmemCarveoutMaxShared));
    cudaGetLastError();   // a refused hint is not an error of the launch
    g_carve_done.emplace_back(kern, dev);
}

// Launch with programmatic stream serialization: the kernel may start while
// the previous kernel on the stream drains; the kernels order their own
// global reads with griddepcontrol.wait.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args&&... args) {
    uniform_carveout(reinterpret_cast<const void*>(kern));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// The same with thread-block clusters of `cluster_x` CTAs along x.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl_cluster(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, int cluster_x,
                               cudaStream_t s, Args&&... args) {
    uniform_carveout(reinterpret_cast<const void*>(kern));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = unsigned(cluster_x);
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// ---------------------------------------------------------------------------
// helpers
// ---------------------------------------------------------------------------
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }
inline size_t elem_bytes(int dtype) { return dtype == MOE_BF16 ? 2 : 4; }
inline int ceil_div(long long a, long long b) { return int((a + b - 1) / b); }

// CTA-pair FFN tiles: the heuristic's choice unless the environment
// variable MOE_PAIR_TILES is "0" (never) or "1" (always)
bool pair_tiles_enabled(bool heuristic) {
    static const int forced = []() {
        const char* v = std::getenv("MOE_PAIR_TILES");
        if (v == nullptr || *v == 0) return -1;
        return v[0] == '0' ? 0 : 1;
    }();
    return forced < 0 ? heuristic : forced == 1;
}

// fc1 on CTA pairs as well: the heuristic's choice unless MOE_FC1_PAIRS is
// "0" (never) or "1" (always)
bool fc1_pair_tiles_enabled(bool heuristic) {
    static const int forced = []() {
        const char* v = std::getenv("MOE_FC1_PAIRS");
        if (v == nullptr || *v == 0) return -1;
        return v[0] == '0' ? 0 : 1;
    }();
    return forced < 0 ? heuristic : forced == 1;
}

// Hot/cold interleaved tile walk in the grouped FFN (decode_tile): the
// heuristic's choice unless MOE_TILE_ZIP is "0" (never) or "1" (always)
bool tile_zip_enabled(bool heuristic) {
    static const int forced = []() {
        const char* v = std::getenv("MOE_TILE_ZIP");
        if (v == nullptr || *v == 0) return -1;
        return v[0] == '0' ? 0 : 1;
    }();
    return forced < 0 ? heuristic : forced == 1;
}

int num_sms() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
    return n;
}

// shared size checks: returns MOE_OK or an error code
int check_sizes(int T, int d, int ff, int E, int k, int dtype, bool need_ff) {
    if (T < 0 || d <= 0 || E <= 0 || k <= 0 || (need_ff && ff <= 0)) return MOE_ERR_INVALID_ARG;
    if (k > E) return MOE_ERR_INVALID_ARG;
    if (dtype != MOE_F32 && dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
    if (E > MOE_MAX_EXPERTS || k > MOE_MAX_TOPK) return MOE_ERR_UNSUPPORTED;
    if (d % 8 != 0 || (need_ff && ff % 8 != 0)) return MOE_ERR_UNSUPPORTED;
    if (static_cast<long long>(T) * k >= (1ll << 31)) return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

int check_shared(int T, int k, int S) {
    if (S < 0) return MOE_ERR_INVALID_ARG;
    if (S > MOE_MAX_SHARED) return MOE_ERR_UNSUPPORTED;
    if (static_cast<long long>(T) * (k + S) >= (1ll << 31)) return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

// F rerouting rounds need k + F distinct experts per token
int check_reroute(int k, int E, int F) {
    if (F < 0) return MOE_ERR_INVALID_ARG;
    if (k + F > MOE_MAX_TOPK) return MOE_ERR_UNSUPPORTED;
    if (k + F > E) return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

// bf16 tensor-core GEMM tile: 128 x 256 (the widest single-CTA MMA; narrower
// tiles measured slower on every workload: more A re-reads per FLOP)
constexpr int kTcBN = 256, kTcStages = 4;
// fc1's GELU epilogue runs on 16 warps (four per TMEM lane quarter) so that
// it keeps pace with the main loop at short K; fc2's bias-and-gate epilogue
// needs only 8
constexpr int kTcFc1EpiWarps = 16;
// Scratch of a rerouting dispatch (F rounds, nchunk chunks).
struct RerouteWs {
    int32_t* srv;     // [T*k]
    int32_t* srank;   // [T*k]
    int32_t* otok;    // [T]
    int32_t* orank;   // [T]
    int32_t* rhist;   // [nchunk][E]
    int32_t* rbase;   // [F][nchunk][E]
    int32_t* load;    // [E]
    int32_t* acc;     // [F][E]
    int32_t* start;   // [F][E]
};

size_t reroute_ws_bytes(int T, int k, int E, int F, int nchunk) {
    const size_t A = size_t(T) * k;
    return align256(A * 4) * 2 + align256(size_t(T) * 4) * 2 + align256(size_t(nchunk) * E * 4) +
           align256(size_t(F) * nchunk * E * 4) + align256(size_t(E) * 4) + align256(size_t(F) * E * 4) * 2;
}

RerouteWs carve_reroute_ws(void* base, int T, int k, int E, int F, int nchunk) {
    uint8_t* p = static_cast<uint8_t*>(base);
    auto take = [&](size_t bytes) {
        int32_t* r = reinterpret_cast<int32_t*>(p);
        p += align256(bytes);
        return r;
    };
    const size_t A = size_t(T) * k;
    RerouteWs w;
    w.srv = take(A * 4);
    w.srank = take(A * 4);
    w.otok = take(size_t(T) * 4);
    w.orank = take(size_t(T) * 4);
    w.rhist = take(size_t(nchunk) * E * 4);
    w.rbase = take(size_t(F) * nchunk * E * 4);
    w.load = take(size_t(E) * 4);
    w.acc = take(size_t(F) * E * 4);
    w.start = take(size_t(F) * E * 4);
    return w;
}

struct WsLayout {
    size_t idx, gate, counts, offsets, perm, slot_of, row_gate, xp, h, yp;
    size_t fhist, fbase, fpsum;   // per-router-chunk arrays of the forward path
    size_t fb_idx, fb_gate, reroute;   // overflow rerouting (F > 0)
    size_t total;
};

// tokens per router CTA (= one dispatch chunk of the forward path)
// Tokens per router CTA (= one dispatch chunk of the forward path).  bf16
// uses 128-token tiles (32- and 64-token tiles and a split-K cluster of 4
// CTAs per tile were measured no faster: every router CTA pays the same
// fixed load -> MMA -> epilogue chain).
inline int router_chunk_tokens(int dtype) { return dtype == MOE_BF16 ? kRtBM : kRouterTM; }

size_t dispatch_ws_bytes(int A, int E) {
    const int nblk = std::max(1, ceil_div(A, kDispChunk));
    return 2 * align256(size_t(nblk) * E * sizeof(int32_t));
}

// S shared experts add S * T rows to h and yp, after the T * k routed rows;
// F rerouting rounds add the fallback lists and the rerouting scratch
WsLayout ws_layout(int T, int d, int ff, int E, int k, int dtype, int S = 0, int F = 0) {
    WsLayout L{};
    const size_t A = size_t(T) * k, es = elem_bytes(dtype);
    const size_t HR = A + size_t(S) * T;   // rows of h and yp
    size_t o = 0;
    auto take = [&](size_t bytes) {
        const size_t r = o;
        o += align256(std::max<size_t>(bytes, 1));
        return r;
    };
    L.idx = take(A * 4);
    L.gate = take(A * 4);
    L.counts = take(size_t(E) * 4);
    L.offsets = take(size_t(E + 1) * 4);
    L.perm = take(A * 4);
    L.slot_of = take(A * 4);
    L.row_gate = take(A * 4);
    L.xp = take(A * d * es);
    L.h = take(HR * ff * es);
    L.yp = take(HR * d * es);
    const size_t nchunk = size_t(std::max(1, ceil_div(T, router_chunk_tokens(dtype))));
    L.fhist = take(nchunk * E * 4);
    L.fbase = take(nchunk * E * 4);
    L.fpsum = take(nchunk * E * 4);
    L.fb_idx = take(size_t(T) * F * 4);
    L.fb_gate = take(size_t(T) * F * 4);
    L.reroute = take(F > 0 ? reroute_ws_bytes(T, k, E, F, int(nchunk)) : 0);
    L.total = o;
    return L;
}

// ---------------------------------------------------------------------------
// TMA tensor maps (driver entry point fetched through the runtime, so the
// library does not link libcuda directly)
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = []() -> EncodeTiledFn {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        return reinterpret_cast<EncodeTiledFn>(p);
    }();
    return fn;
}

// [rows, cols] row-major of dtype (bf16 or fp32), box {128 B of columns,
// box_rows}, 128B swizzle
bool make_map_2d(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint32_t box_rows,
                 int dtype = MOE_BF16) {
    EncodeTiledFn enc = encode_fn();
    if (enc == nullptr) return false;
    const uint64_t es = elem_bytes(dtype);
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * es};
    const cuuint32_t box[2] = {uint32_t(128 / es), box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, dtype == MOE_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2,
               const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [E, rows, cols] of dtype, box {128 B of columns, box_rows, 1}, 128B swizzle
bool make_map_3d(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint64_t E, uint32_t box_rows,
                 int dtype = MOE_BF16) {
    EncodeTiledFn enc = encode_fn();
    if (enc == nullptr) return false;
    const uint64_t es = elem_bytes(dtype);
    const cuuint64_t dims[3] = {cols, rows, E};
    const cuuint64_t strides[2] = {cols * es, cols * rows * es};
    const cuuint32_t box[3] = {uint32_t(128 / es), box_rows, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, dtype == MOE_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3,
               const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The grouped FFN's output C [rows, cols] bf16 for the epilogue's TMA
// tile stores: box {seg_bytes / 2 columns, 32 rows}, the swizzle whose
// span equals the box's row (64 or 32 bytes)
bool make_store_map(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint32_t seg_bytes) {
    EncodeTiledFn enc = encode_fn();
    if (enc == nullptr) return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * 2};
    const cuuint32_t box[2] = {seg_bytes / 2, 32};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, seg_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B,
               CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Raises a kernel's dynamic shared memory limit once per device (later
// calls, e.g. while a CUDA graph is being captured, only look it up).
std::mutex g_attr_mu;
std::vector<std::pair<const void*, int>> g_attr_done;   // (kernel, device) already set

template <typename K>
bool set_smem_attr(K kernel, size_t bytes) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    const void* key = reinterpret_cast<const void*>(kernel);
    std::lock_guard<std::mutex> lk(g_attr_mu);
    for (const auto& kd : g_attr_done)
        if (kd.first == key && kd.second == dev) return true;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(bytes)) != cudaSuccess)
        return false;
    g_attr_done.emplace_back(key, dev);
    return true;
}

// CTAs of `kernel` (`threads` per CTA, no dynamic shared memory) that fit on
// one SM at once; cached per (kernel, device); 1 if the query fails.
std::mutex g_occ_mu;
std::vector<std::pair<std::pair<const void*, int>, int>> g_occ_done;

template <typename K>
int resident_blocks(K kernel, int threads) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return 1;
    const void* key = reinterpret_cast<const void*>(kernel);
    std::lock_guard<std::mutex> lk(g_occ_mu);
    for (const auto& kd : g_occ_done)
        if (kd.first.first == key && kd.first.second == dev) return kd.second;
    uniform_carveout(key);
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, threads, 0) != cudaSuccess || n < 1) {
        cudaGetLastError();
        n = 1;
    }
    g_occ_done.push_back({{key, dev}, n});
    return n;
}

// ---------------------------------------------------------------------------
// step launchers (arguments already validated)
// ---------------------------------------------------------------------------
// F > 0: also the next F experts of each token (fallbacks for overflow
// rerouting) into fb_idx / fb_gate [T, F]
struct RouterOut {
    int32_t* idx;
    float* gate;
    float* psum;        // [E] atomic sums (zeroed here), or null
    float* psum_part;   // [tiles][E] per-tile sums, or null
    int32_t* hist;      // [tiles][E] per-tile histograms, or null
    int F;
    int32_t* fb_idx;
    float* fb_gate;
};

template <typename Tin, int EP>
int launch_router_ep(const void* x, const void* wr, const float* bias, int T, int d, int E, int k,
                     const RouterOut& o, cudaStream_t s) {
    auto kern = router_topk_kernel<Tin, EP>;
    const size_t smem = router_smem_bytes<EP>();
    if (!set_smem_attr(kern, smem)) return MOE_ERR_CUDA;
    Launch L(MOE_KERNEL_ROUTER, s);
    cudaError_t launch_err;
    launch_err = launch_pdl(kern, dim3(ceil_div(T, kRouterTM)), dim3(kRouterThreads), smem, s,
                            static_cast<const Tin*>(x), static_cast<const Tin*>(wr), bias, T, d, E, k, o.idx, o.gate,
                            o.psum, o.psum_part, o.hist, o.F, o.fb_idx, o.fb_gate);
    return L.finish(launch_err);
}

// SPLIT = 2: clusters of two CTAs share each 128-token tile's K stages
template <int EP, int KMAX, int SPLIT>
int launch_router_tc(const void* x, const void* wr, const float* bias, int T, int d, int E, int k,
                     const RouterOut& o, cudaStream_t s) {
    CUtensorMap tmX, tmW;
    if (!make_map_2d(&tmX, x, uint64_t(d), uint64_t(T), kRtBM)) return MOE_ERR_UNSUPPORTED;
    if (!make_map_2d(&tmW, wr, uint64_t(d), uint64_t(E), EP)) return MOE_ERR_UNSUPPORTED;
    auto kern = router_tc_kernel<EP, KMAX, SPLIT>;
    const size_t smem = RtCfg<EP, SPLIT>::kSmemBytes;
    if (!set_smem_attr(kern, smem)) return MOE_ERR_CUDA;
    const int tiles = ceil_div(T, kRtBM);
    Launch L(MOE_KERNEL_ROUTER, s);
    cudaError_t launch_err;
    if (SPLIT == 2)
        launch_err = launch_pdl_cluster(kern, dim3(2 * tiles), dim3(kRtThreads), smem, 2, s, tmX, tmW, bias, T, d, E,
                                        k, o.idx, o.gate, o.psum, o.psum_part, o.hist, o.F, o.fb_idx, o.fb_gate);
    else
        launch_err = launch_pdl(kern, dim3(tiles), dim3(kRtThreads), smem, s, tmX, tmW, bias, T, d, E, k, o.idx,
                                o.gate, o.psum, o.psum_part, o.hist, o.F, o.fb_idx, o.fb_gate);
    return L.finish(launch_err);
}

// The K split over two CTAs per tile when the tiles leave half the SMs idle
// and each CTA still gets eight or more K stages (large d, few tokens:
// large-top2 runs 64 tiles of 64 stages), for up to 64 experts.
template <int KMAX>
int launch_router_tc_k(const void* x, const void* wr, const float* bias, int T, int d, int E, int k,
                       const RouterOut& o, cudaStream_t s) {
    const bool split = 2 * ceil_div(T, kRtBM) <= num_sms() && ceil_div(d, 64) >= 16;
    if (E <= 16)
        return split ? launch_router_tc<16, KMAX, 2>(x, wr, bias, T, d, E, k, o, s)
                     : launch_router_tc<16, KMAX, 1>(x, wr, bias, T, d, E, k, o, s);
    if (E <= 32)
        return split ? launch_router_tc<32, KMAX, 2>(x, wr, bias, T, d, E, k, o, s)
                     : launch_router_tc<32, KMAX, 1>(x, wr, bias, T, d, E, k, o, s);
    if (E <= 64)
        return split ? launch_router_tc<64, KMAX, 2>(x, wr, bias, T, d, E, k, o, s)
                     : launch_router_tc<64, KMAX, 1>(x, wr, bias, T, d, E, k, o, s);
    if (E <= 128) return launch_router_tc<128, KMAX, 1>(x, wr, bias, T, d, E, k, o, s);
    return launch_router_tc<256, KMAX, 1>(x, wr, bias, T, d, E, k, o, s);
}

template <typename Tin>
int launch_router_t(const void* x, const void* wr, const float* bias, int T, int d, int E, int k,
                    const RouterOut& o, cudaStream_t s) {
    if (E <= 16) return launch_router_ep<Tin, 16>(x, wr, bias, T, d, E, k, o, s);
    if (E <= 32) return launch_router_ep<Tin, 32>(x, wr, bias, T, d, E, k, o, s);
    if (E <= 64) return launch_router_ep<Tin, 64>(x, wr, bias, T, d, E, k, o, s);
    if (E <= 128) return launch_router_ep<Tin, 128>(x, wr, bias, T, d, E, k, o, s);
    return launch_router_ep<Tin, 256>(x, wr, bias, T, d, E, k, o, s);
}

// bf16: tcgen05 router (128-token tiles); f32: SIMT fp32 router (32-token
// tiles).  prob_sum (atomic, zeroed here) or psum_part/hist (per tile) as
// requested in `o`.
int run_router(const void* x, const void* wr, const float* bias, int T, int d, int E, int k, int dtype,
               const RouterOut& o, cudaStream_t s) {
    if (o.psum != nullptr && o.psum_part == nullptr &&
        cudaMemsetAsync(o.psum, 0, size_t(E) * sizeof(float), s) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (dtype == MOE_BF16) {
        const int ksel = k + o.F;
        if (ksel == 1) return launch_router_tc_k<1>(x, wr, bias, T, d, E, k, o, s);
        if (ksel == 2) return launch_router_tc_k<2>(x, wr, bias, T, d, E, k, o, s);
        return launch_router_tc_k<MOE_MAX_TOPK>(x, wr, bias, T, d, E, k, o, s);
    }
    return launch_router_t<float>(x, wr, bias, T, d, E, k, o, s);
}

int run_dispatch(const int32_t* idx, const float* gate, int T, int k, int E, int capacity, int32_t* counts,
                 int32_t* offsets, int32_t* perm, int32_t* slot_of, uint8_t* drop, float* row_gate, const void* x,
                 void* xp, int d, int dtype, void* ws, cudaStream_t s) {
    const int A = T * k;
    const int nblk = ceil_div(A, kDispChunk);
    int32_t* hist = static_cast<int32_t*>(ws);
    int32_t* base = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(ws) + dispatch_ws_bytes(A, E) / 2);
    int rc;
    {
        Launch L(MOE_KERNEL_COUNT, s);
        cudaError_t launch_err;
        launch_err = launch_pdl(dispatch_count_kernel, dim3(nblk), dim3(kDispThreads), 0, s, idx, A, E, hist);
        if ((rc = L.finish(launch_err)) != MOE_OK) return rc;
    }
    {
        Launch L(MOE_KERNEL_SCAN, s);
        cudaError_t launch_err;
        launch_err = launch_pdl(dispatch_scan_kernel, dim3(1), dim3(kDispThreads), 0, s, hist, nblk, E, capacity, base, counts, offsets);
        if ((rc = L.finish(launch_err)) != MOE_OK) return rc;
    }
    {
        Launch L(MOE_KERNEL_PERMUTE, s);
        cudaError_t launch_err;
        launch_err = launch_pdl(dispatch_permute_kernel, dim3(nblk), dim3(kDispThreads), 0, s, idx, gate, A, E, base, offsets, perm, slot_of, drop,
                                                               row_gate);
        if ((rc = L.finish(launch_err)) != MOE_OK) return rc;
    }
    if (x != nullptr && xp != nullptr) {
        const int row_bytes = int(size_t(d) * elem_bytes(dtype));
        const int grid = std::max(1, std::min(ceil_div(A, 8), num_sms() * 8));
        Launch L(MOE_KERNEL_GATHER, s);
        cudaError_t launch_err;
        launch_err = launch_pdl(dispatch_gather_kernel, dim3(grid), dim3(256), 0, s, static_cast<const uint8_t*>(x), row_bytes, perm, offsets, E, k,
                                                    static_cast<uint8_t*>(xp), static_cast<const int32_t*>(nullptr), 0, static_cast<uint8_t*>(nullptr));
        if ((rc = L.finish(launch_err)) != MOE_OK) return rc;
    }
    return MOE_OK;
}


// The shared always-on experts of one FFN GEMM (host side): S groups of
// `g.rows` rows each, A rows from `a` (a_rows rows in all), weights [S, N, K]
// and biases [S, N].  S = 0: none.
struct SharedArgs {
    const void* a = nullptr;
    int a_rows = 0;
    const void* w = nullptr;
    const void* bias = nullptr;
    SharedGroups g{};
};

// The four operand maps of a grouped-FFN launch: routed A rows and weights,
// shared-expert A rows and weights (each side falls back to the other when
// it has no groups, so every map handed to the kernel is valid).
struct FfnMaps {
    CUtensorMap a, b, a2, b2;
};

bool make_ffn_maps(FfnMaps& m, const void* a, int a_cols, int a_rows, const void* w, int N, int E,
                   const SharedArgs& sa, uint32_t a_box_rows, uint32_t w_box_rows, int dtype) {
    if (sa.g.S > 0) {
        if (!make_map_2d(&m.a2, sa.a, uint64_t(a_cols), uint64_t(sa.a_rows), a_box_rows, dtype)) return false;
        if (!make_map_3d(&m.b2, sa.w, uint64_t(a_cols), uint64_t(N), uint64_t(sa.g.S), w_box_rows, dtype))
            return false;
    }
    if (E > 0) {
        if (!make_map_2d(&m.a, a, uint64_t(a_cols), uint64_t(a_rows), a_box_rows, dtype)) return false;
        if (!make_map_3d(&m.b, w, uint64_t(a_cols), uint64_t(N), uint64_t(E), w_box_rows, dtype)) return false;
    } else {
        m.a = m.a2;
        m.b = m.b2;
    }
    if (sa.g.S == 0) {
        m.a2 = m.a;
        m.b2 = m.b;
    }
    return true;
}

// Upper bound of a launch's tiles (the real count comes from the device offsets)
long long ffn_tiles_ub(int routed_rows_ub, int E, const SharedArgs& sa, int BM, int N, int BN) {
    const long long mt_ub = static_cast<long long>(ceil_div(routed_rows_ub, BM)) + E +
                            static_cast<long long>(sa.g.S) * ceil_div(sa.g.rows, BM);
    return mt_ub * ceil_div(N, BN);
}

// Routed groups: E experts over rows offsets[0..E] of `a` (a_rows rows;
// routed_rows_ub bounds offsets[E]).  E may be 0 when only shared groups run.

template <int BN, int STAGES, int MODE, int EPIW = kTcEpiWarps>
int launch_tc(const void* a, int a_cols, int a_rows, int routed_rows_ub, const void* w, int N, int E,
              const int32_t* offsets, const void* bias, const float* row_gate, const int32_t* out_rows, void* c,
              int c_rows, const SharedArgs& sa, int kernel_id, cudaStream_t s, bool zip = false) {
    FfnMaps mp;
    if (!make_ffn_maps(mp, a, a_cols, a_rows, w, N, E, sa, kTcBM, BN, MOE_BF16)) return MOE_ERR_UNSUPPORTED;
    CUtensorMap tmC;
    if (!make_store_map(&tmC, c, uint64_t(N), uint64_t(c_rows), epi_seg_bytes(EPIW))) return MOE_ERR_UNSUPPORTED;
    auto kern = ffn_tc_bf16_kernel<BN, STAGES, MODE, EPIW>;
    const size_t smem = TcCfg<BN, STAGES>::smem_bytes(EPIW);
    if (!set_smem_attr(kern, smem)) return MOE_ERR_CUDA;
    const long long tiles_ub = ffn_tiles_ub(routed_rows_ub, E, sa, kTcBM, N, BN);
    const int grid = int(std::max(1ll, std::min<long long>(tiles_ub, num_sms())));
    Launch L(kernel_id, s);
    cudaError_t launch_err;
    launch_err = launch_pdl(kern, dim3(grid), dim3(tc_threads(EPIW)), smem, s, mp.a, mp.b, offsets, E, N, a_cols,
                            static_cast<const __nv_bfloat16*>(bias), row_gate, out_rows,
                            static_cast<__nv_bfloat16*>(c), sa.g, mp.a2, mp.b2,
                            static_cast<const __nv_bfloat16*>(sa.bias), zip ? 1 : 0, tmC, out_rows == nullptr ? 1 : 0);
    return L.finish(launch_err);
}

// The CTA-pair variant (cta_group::2, 256 x 256 tiles): A map boxes of 128
// rows, weight map boxes of 128 rows (half of the tile's N).
constexpr int kTc2Stages = 6;

template <int MODE, int EPIW = kTcEpiWarps>
int launch_tc2(const void* a, int a_cols, int a_rows, int routed_rows_ub, const void* w, int N, int E,
               const int32_t* offsets, const void* bias, const float* row_gate, const int32_t* out_rows, void* c,
               int c_rows, const SharedArgs& sa, int kernel_id, cudaStream_t s, bool zip = false) {
    FfnMaps mp;
    if (!make_ffn_maps(mp, a, a_cols, a_rows, w, N, E, sa, 128, kTc2BN / 2, MOE_BF16)) return MOE_ERR_UNSUPPORTED;
    CUtensorMap tmC;
    if (!make_store_map(&tmC, c, uint64_t(N), uint64_t(c_rows), epi_seg_bytes(EPIW))) return MOE_ERR_UNSUPPORTED;
    auto kern = ffn_tc2_bf16_kernel<kTc2Stages, MODE, EPIW>;
    const size_t smem = Tc2Cfg<kTc2Stages>::smem_bytes(EPIW);
    if (!set_smem_attr(kern, smem)) return MOE_ERR_CUDA;
    const long long tiles_ub = ffn_tiles_ub(routed_rows_ub, E, sa, kTc2BM, N, kTc2BN);
    const int pairs = int(std::max(1ll, std::min<long long>(tiles_ub, num_sms() / 2)));
    Launch L(kernel_id, s);
    cudaError_t launch_err;
    launch_err = launch_pdl_cluster(kern, dim3(2 * pairs), dim3(tc_threads(EPIW)), smem, 2, s, mp.a, mp.b, offsets, E, N,
                                    a_cols, static_cast<const __nv_bfloat16*>(bias), row_gate, out_rows,
                                    static_cast<__nv_bfloat16*>(c), sa.g, mp.a2, mp.b2,
                                    static_cast<const __nv_bfloat16*>(sa.bias), zip ? 1 : 0, tmC,
                                    out_rows == nullptr ? 1 : 0);
    return L.finish(launch_err);
}

// fp32 on the tensor cores, three-pass TF32: 128 x 128 tiles, 4 stages
constexpr int kTfBN = 128, kTfStages = 4;

template <int MODE>
int launch_tf32x3(const void* a, int a_cols, int a_rows, int routed_rows_ub, const void* w, int N, int E,
                  const int32_t* offsets, const void* bias, const float* row_gate, const int32_t* out_rows, void* c,
                  const SharedArgs& sa, int kernel_id, cudaStream_t s, bool zip = false) {
    FfnMaps mp;
    if (!make_ffn_maps(mp, a, a_cols, a_rows, w, N, E, sa, kTcBM, kTfBN, MOE_F32)) return MOE_ERR_UNSUPPORTED;
    auto kern = ffn_tc_f32x3_kernel<kTfBN, kTfStages, MODE>;
    const size_t smem = TfCfg<kTfBN, kTfStages>::kSmemBytes;
    if (!set_smem_attr(kern, smem)) return MOE_ERR_CUDA;
    const long long tiles_ub = ffn_tiles_ub(routed_rows_ub, E, sa, kTcBM, N, kTfBN);
    const int grid = int(std::max(1ll, std::min<long long>(tiles_ub, num_sms())));
    Launch L(kernel_id, s);
    cudaError_t launch_err;
    launch_err = launch_pdl(kern, dim3(grid), dim3(kTfThreads), smem, s, mp.a, mp.b, offsets, E, N, a_cols,
                            static_cast<const float*>(bias), row_gate, out_rows, static_cast<float*>(c), sa.g, mp.a2,
                            mp.b2, static_cast<const float*>(sa.bias), zip ? 1 : 0);
    return L.finish(launch_err);
}

// The shared experts of a layer (S = 0: none): parameters [S, ...] and the
// tokens x [T, d] they read.
struct SharedExperts {
    int S = 0;
    int T = 0;
    const void* x = nullptr;
    const void *w1 = nullptr, *b1 = nullptr, *w2 = nullptr, *b2 = nullptr;
};

// Grouped FFN over the E routed groups (rows offsets[e] .. offsets[e+1]-1 of
// xp, routed rows < max_rows) and the shared experts.  h and yp hold
// max_rows routed rows followed by S * T shared rows (shared expert s, token
// t at row max_rows + s * T + t).  out_rows (nullable): fc2 writes routed
// row r to row out_rows[r] of yp (the direct output of a k == 1 layer).
// fc2 tile width for layers whose experts hold about one 128-row tile each:
// 192 instead of 256 columns when that keeps the expected tiles within one
// wave while 256 would leave a quarter of the SMs idle (expected tiles
// assume balanced experts; the tile table itself comes from the device)
constexpr int kTcBNNarrow = 192, kTcStagesNarrow = 5;

bool fc2_narrow_tiles(int max_rows, int E, int N, const SharedExperts& se) {
    if (E <= 0) return false;
    const long long per_expert = ceil_div(ceil_div(max_rows, E), kTcBM);
    const long long mt = per_expert * E + static_cast<long long>(se.S) * ceil_div(se.T, kTcBM);
    const long long wide = mt * ceil_div(N, kTcBN), narrow = mt * ceil_div(N, kTcBNNarrow);
    const int sms = num_sms();
    return 4 * wide < 3ll * sms && narrow <= sms && narrow > wide;
}

// use_pairs: bf16 fc2 on CTA pairs (256-row tiles), for layers whose experts
// average enough rows that the doubled M tile wastes little
int run_ffn(const void* xp, const int32_t* offsets, int max_rows, int E, int d, int ff, const void* w1,
            const void* b1, const void* w2, const void* b2, const float* row_gate, void* h, void* yp, int dtype,
            const int32_t* out_rows, const SharedExperts& se, bool use_pairs, cudaStream_t s,
            bool fc1_pairs = false) {
    const int h_rows = max_rows + se.S * se.T;
    SharedArgs s1, s2;
    if (se.S > 0) {
        // fc1 of shared expert s: A = x (every shared expert reads the same rows)
        s1.a = se.x;
        s1.a_rows = se.T;
        s1.w = se.w1;
        s1.bias = se.b1;
        s1.g = SharedGroups{se.S, se.T, 0, 0, max_rows};
        // fc2 of shared expert s: A = its rows of h
        s2.a = h;
        s2.a_rows = h_rows;
        s2.w = se.w2;
        s2.bias = se.b2;
        s2.g = SharedGroups{se.S, se.T, max_rows, se.T, max_rows};
    }
    const bool zip = tile_zip_enabled(false);
    int rc;
    if (dtype == MOE_BF16) {
        // fc1 stays on single-CTA 128-row tiles: its K (= d) is short, so the
        // pair kernel's doubled M padding costs more than its halved loads
        // save (measured on the skewed and large workloads)
        if (fc1_pairs)
            rc = launch_tc2<kFc1Gelu, kTcFc1EpiWarps>(xp, d, max_rows, max_rows, w1, ff, E, offsets, b1, nullptr,
                                                      nullptr, h, h_rows, s1, MOE_KERNEL_FFN1, s, zip);
        else
            rc = launch_tc<kTcBN, kTcStages, kFc1Gelu, kTcFc1EpiWarps>(xp, d, max_rows, max_rows, w1, ff, E,
                                                                       offsets, b1, nullptr, nullptr, h, h_rows,
                                                                       s1, MOE_KERNEL_FFN1, s, zip);
        if (rc != MOE_OK) return rc;
        // yp's rows for the epilogue's TMA stores (h_rows; with out_rows the
        // kernels store row by row and never use that map)
        if (use_pairs)
            return launch_tc2<kFc2Gate>(h, ff, h_rows, max_rows, w2, d, E, offsets, b2, row_gate, out_rows, yp,
                                        h_rows, s2, MOE_KERNEL_FFN2, s, zip);
        // fc2 of a layer with about one M tile per expert (switch-top1: 96
        // tiles of 256 columns for 148 SMs): 192-column tiles put 4/3 as many
        // SMs on the weight stream
        if (fc2_narrow_tiles(max_rows, E, d, se))
            return launch_tc<kTcBNNarrow, kTcStagesNarrow, kFc2Gate>(h, ff, h_rows, max_rows, w2, d, E, offsets, b2,
                                                                     row_gate, out_rows, yp, h_rows, s2, MOE_KERNEL_FFN2, s,
                                                                     zip);
        return launch_tc<kTcBN, kTcStages, kFc2Gate>(h, ff, h_rows, max_rows, w2, d, E, offsets, b2, row_gate,
                                                     out_rows, yp, h_rows, s2, MOE_KERNEL_FFN2, s, zip);
    }
    rc = launch_tf32x3<kFc1Gelu>(xp, d, max_rows, max_rows, w1, ff, E, offsets, b1, nullptr, nullptr, h, s1,
                                 MOE_KERNEL_FFN1, s, zip);
    if (rc != MOE_OK) return rc;
    return launch_tf32x3<kFc2Gate>(h, ff, h_rows, max_rows, w2, d, E, offsets, b2, row_gate, out_rows, yp, s2,
                                   MOE_KERNEL_FFN2, s, zip);
}

// Dispatch of the fused forward path from the router's per-chunk histograms
// and probability sums: one scan CTA (+ statistics), then the permute /
// gather kernel over (chunk, G) CTAs.
int permute_split(int nchunk) { return std::max(1, std::min(8, ceil_div(2 * num_sms(), nchunk))); }

// the fused scan + permute kernel reads the whole per-chunk histogram table
// in every CTA: used while that table is small
constexpr long long kFusedScanMaxEntries = 16384;

int run_forward_dispatch(const int32_t* idx, const float* gate, int T, int k, int E, int capacity, int chunk_tokens,
                         const int32_t* fhist, const float* fpsum, int32_t* fbase, int32_t* counts, int32_t* offsets,
                         int32_t* perm, int32_t* slot_of, uint8_t* drop_mask, float* row_gate, moe_stats* st,
                         const void* x, void* xp, int d, int dtype, void* out_zero_dropped, cudaStream_t s) {
    const int nchunk = ceil_div(T, chunk_tokens);
    int rc;
    if (drop_mask == nullptr && static_cast<long long>(nchunk) * E <= kFusedScanMaxEntries) {
        const int row_bytes = int(size_t(d) * elem_bytes(dtype));
        // the row gather on bulk copies through a ring of row buffers, for
        // rows of at least kGatherBulkMinRow bytes (below that one issuing
        // thread's per-row overhead outweighs the copies: the thread-wide
        // 16-byte gather is faster), when every address is 16-byte aligned
        // and the ring holds enough rows
        const int zero_bytes = out_zero_dropped != nullptr ? row_bytes : 0;
        int ring_rows = 0;
        if (x != nullptr && xp != nullptr && row_bytes >= kGatherBulkMinRow && row_bytes % 16 == 0 &&
            aligned16(x) && aligned16(xp) &&
            (out_zero_dropped == nullptr || aligned16(out_zero_dropped)) && row_bytes <= int(kGatherSmem)) {
            ring_rows = std::min(kGatherRing, int((kGatherSmem - uint32_t(zero_bytes)) / uint32_t(row_bytes)));
            if (ring_rows < kGatherLag + 1) ring_rows = 0;
        }
        const size_t dyn = ring_rows > 0 ? size_t(ring_rows) * row_bytes + zero_bytes : 0;
        if (dyn > 0 && !set_smem_attr(forward_dispatch_kernel, size_t(kGatherSmem))) return MOE_ERR_CUDA;
        Launch L(MOE_KERNEL_PERMUTE, s);
        cudaError_t launch_err;
        launch_err = launch_pdl(forward_dispatch_kernel, dim3(nchunk, permute_split(nchunk)), dim3(kFwdThreads), dyn,
                                s, idx, gate, T, k, E, chunk_tokens, fhist, fpsum, nchunk, capacity, counts, offsets,
                                st, perm, slot_of, row_gate, static_cast<const uint8_t*>(x), row_bytes,
                                static_cast<uint8_t*>(xp), static_cast<uint8_t*>(out_zero_dropped), ring_rows);
        return L.finish(launch_err);
    }
    {
        Launch L(MOE_KERNEL_SCAN, s);
        cudaError_t launch_err;
        launch_err = launch_pdl(forward_scan_kernel, dim3(1), dim3(kFwdScanThreads), 0, s, fhist, fpsum, nchunk, E,
                                T, k, capacity, fbase, counts, offsets, st, static_cast<int32_t*>(nullptr));
        if ((rc = L.finish(launch_err)) != MOE_OK) return rc;
    }
    const int row_bytes = int(size_t(d) * elem_bytes(dtype));
    Launch L(MOE_KERNEL_PERMUTE, s);
    cudaError_t launch_err;
    launch_err = launch_pdl(forward_permute_kernel, dim3(nchunk, permute_split(nchunk)), dim3(kFwdThreads), 0, s,
                            idx, gate, T, k, E, chunk_tokens, fbase, offsets, perm, slot_of, row_gate,
                            static_cast<const uint8_t*>(x), row_bytes, static_cast<uint8_t*>(xp),
                            static_cast<uint8_t*>(out_zero_dropped), drop_mask);
    return L.finish(launch_err);
}

// Dispatch with F >= 1 rerouting rounds (capacity >= 0), from per-chunk
// histograms of the own choices: scan, F x (mark, scan), permute / gather.
int run_reroute_dispatch(const int32_t* idx, const float* gate, const int32_t* fb_idx, const float* fb_gate, int T,
                         int k, int E, int capacity, int F, int chunk_tokens, const int32_t* fhist,
                         const float* fpsum, int32_t* fbase, int32_t* counts, int32_t* offsets, int32_t* perm,
                         int32_t* slot_of, uint8_t* drop_mask, float* row_gate, moe_stats* st, const void* x,
                         void* xp, int d, int dtype, void* out_zero_dropped, const RerouteWs& rw, cudaStream_t s) {
    const int nchunk = ceil_div(T, chunk_tokens);
    const size_t ce = size_t(nchunk) * E;
    int rc;
    {
        Launch L(MOE_KERNEL_SCAN, s);
        cudaError_t launch_err;
        launch_err = launch_pdl(forward_scan_kernel, dim3(1), dim3(kFwdScanThreads), 0, s, fhist, fpsum, nchunk, E,
                                T, k, capacity, fbase, counts, offsets, st, rw.load);
        if ((rc = L.finish(launch_err)) != MOE_OK) return rc;
    }
    for (int r = 1; r <= F; ++r) {
        {
            Launch L(MOE_KERNEL_REROUTE, s);
            cudaError_t launch_err;
            const int32_t* prev_rbase = r > 1 ? rw.rbase + size_t(r - 2) * ce : nullptr;
            const int32_t* prev_acc = r > 1 ? rw.acc + size_t(r - 2) * E : nullptr;
            launch_err = launch_pdl(reroute_mark_kernel, dim3(nchunk), dim3(kFwdThreads), 0, s, idx, T, k, E,
                                    chunk_tokens, capacity, static_cast<const int32_t*>(fbase), fb_idx, F, r,
                                    prev_rbase, prev_acc, rw.srv, rw.srank, rw.otok, rw.orank, rw.rhist);
            if ((rc = L.finish(launch_err)) != MOE_OK) return rc;
        }
        {
            Launch L(MOE_KERNEL_REROUTE, s);
            cudaError_t launch_err;
            launch_err = launch_pdl(reroute_scan_kernel, dim3(1), dim3(kFwdScanThreads), 0, s,
                                    static_cast<const int32_t*>(rw.rhist), nchunk, E, capacity, r, F, T, k,
                                    rw.rbase + size_t(r - 1) * ce, rw.load, rw.acc + size_t(r - 1) * E,
                                    rw.start + size_t(r - 1) * E, offsets, st);
            if ((rc = L.finish(launch_err)) != MOE_OK) return rc;
        }
    }
    const int row_bytes = int(size_t(d) * elem_bytes(dtype));
    Launch L(MOE_KERNEL_PERMUTE, s);
    cudaError_t launch_err;
    launch_err = launch_pdl(reroute_permute_kernel, dim3(nchunk, permute_split(nchunk)), dim3(kFwdThreads), 0, s,
                            idx, gate, fb_idx, fb_gate, T, k, E, F, chunk_tokens,
                            static_cast<const int32_t*>(rw.srv), static_cast<const int32_t*>(rw.srank),
                            static_cast<const int32_t*>(rw.otok), static_cast<const int32_t*>(rw.orank),
                            static_cast<const int32_t*>(rw.rbase + size_t(F - 1) * ce),
                            static_cast<const int32_t*>(rw.acc + size_t(F - 1) * E),
                            static_cast<const int32_t*>(rw.start), static_cast<const int32_t*>(offsets), perm,
                            slot_of, row_gate, static_cast<const uint8_t*>(x), row_bytes, static_cast<uint8_t*>(xp),
                            static_cast<uint8_t*>(out_zero_dropped), drop_mask);
    return L.finish(launch_err);
}

// ys (nullable when S == 0): [S, T, d] shared-expert outputs added with weight 1
int run_combine(const void* yp, const int32_t* slot_of, const float* gate, int T, int k, int d, int dtype, void* out,
                const void* ys, int S, cudaStream_t s) {
    // warps stride over the tokens: no more CTAs than fit on the GPU at once
    const int per_sm = dtype == MOE_BF16 ? resident_blocks(combine_kernel<__nv_bfloat16>, 256)
                                         : resident_blocks(combine_kernel<float>, 256);
    const int grid = std::max(1, std::min(ceil_div(T, 8), num_sms() * per_sm));
    Launch L(MOE_KERNEL_COMBINE, s);
    cudaError_t launch_err;
    if (dtype == MOE_BF16)
        launch_err = launch_pdl(combine_kernel<__nv_bfloat16>, dim3(grid), dim3(256), 0, s,
                                static_cast<const __nv_bfloat16*>(yp), slot_of, gate, T, k, d,
                                static_cast<__nv_bfloat16*>(out), static_cast<const __nv_bfloat16*>(ys), S);
    else
        launch_err = launch_pdl(combine_kernel<float>, dim3(grid), dim3(256), 0, s, static_cast<const float*>(yp),
                                slot_of, gate, T, k, d, static_cast<float*>(out), static_cast<const float*>(ys), S);
    return L.finish(launch_err);
}

int run_stats(const int32_t* counts, const int32_t* offsets, const float* psum, int T, int k, int E, moe_stats* st,
              cudaStream_t s) {
    Launch L(MOE_KERNEL_STATS, s);
    cudaError_t launch_err;
    launch_err = launch_pdl(stats_kernel, dim3(1), dim3(256), 0, s, counts, offsets, psum, T, k, E, st);
    return L.finish(launch_err);
}

// ---------------------------------------------------------------------------
// Fixed device scratch for moe_dispatch_noalloc.  Sized for
// MOE_NOALLOC_MAX_ASSIGNMENTS assignments and MOE_MAX_EXPERTS experts: the
// per-chunk histograms and bases of the dispatch kernels (1 MiB).  Every GPU
// that loads the library holds this array until the process exits.  In host
// code `g_dispatch_scratch` is only a host-side stand-in for the symbol;
// its device address comes from cudaGetSymbolAddress, once per device.
// ---------------------------------------------------------------------------
constexpr size_t kNoallocScratchBytes =
    2 * ((size_t(MOE_NOALLOC_MAX_ASSIGNMENTS) / kDispChunk) * MOE_MAX_EXPERTS * sizeof(int32_t));
static __device__ __align__(256) uint8_t g_dispatch_scratch[kNoallocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};
CUcontext g_noalloc_ctx[kMaxDevices] = {};

// The driver's cuCtxGetCurrent, reached through the runtime (the library
// does not link the driver library); null if the driver does not offer it.
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
CtxGetCurrentFn ctx_get_current() {
    static const CtxGetCurrentFn fn = []() -> CtxGetCurrentFn {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        return reinterpret_cast<CtxGetCurrentFn>(p);
    }();
    return fn;
}

CUcontext current_context() {
    CUcontext c = nullptr;
    const CtxGetCurrentFn f = ctx_get_current();
    if (f == nullptr || f(&c) != CUDA_SUCCESS) return nullptr;
    return c;
}

// Device address of g_dispatch_scratch on the current device, looked up
// with that device current on the first call for it and kept with the
// context it belongs to.  A device reset or a re-created primary context
// gives the device a new context (and the module a new load), so the
// address is looked up again on the next call rather than reused.
int noalloc_scratch(void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
    const CUcontext ctx = current_context();
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (g_noalloc_ptr[dev] == nullptr || ctx == nullptr || ctx != g_noalloc_ctx[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_dispatch_scratch) != cudaSuccess || p == nullptr) return MOE_ERR_CUDA;
        g_noalloc_ptr[dev] = p;
        g_noalloc_ctx[dev] = current_context();   // the runtime has made the context current by now
    }
    *out = g_noalloc_ptr[dev];
    return MOE_OK;
}

}  // namespace

// ===========================================================================
// C ABI
// ===========================================================================
extern "C" {

const char* moe_status_string(int status) {
    switch (status) {
        case MOE_OK: return "ok";
        case MOE_ERR_INVALID_ARG: return "invalid argument";
        case MOE_ERR_UNSUPPORTED: return "unsupported dtype, shape or size";
        case MOE_ERR_WORKSPACE: return "workspace missing or too small";
        case MOE_ERR_CUDA: return "CUDA error";
        case MOE_ERR_BAD_ROUTING: return "expert index out of range";
        case MOE_ERR_TIMEOUT: return "device pipeline wait timed out";
        default: return "unknown status";
    }
}

int moe_version(void) { return 10000; }

int moe_capacity(int T, int k, int E, double cf) {
    if (T < 0 || k < 1 || E < 1) return -1;
    if (!(cf > 0.0)) return -1;
    const double c = double(T) * double(k) / double(E) * cf;
    if (c >= 2147483647.0) return 2147483647;
    return int(c);
}

size_t moe_workspace_size(int T, int d, int ff, int E, int k, int dtype) {
    return moe_forward_ex_workspace_size(T, d, ff, E, k, 0, 0, dtype);
}

size_t moe_forward_ex_workspace_size(int T, int d, int ff, int E, int k, int S, int F, int dtype) {
    if (check_sizes(T, d, ff, E, k, dtype, true) != MOE_OK || check_shared(T, k, S) != MOE_OK ||
        check_reroute(k, E, F) != MOE_OK)
        return 0;
    return ws_layout(T, d, ff, E, k, dtype, S, F).total;
}

size_t moe_workspace_offset(int T, int d, int ff, int E, int k, int dtype, int which) {
    return moe_forward_ex_workspace_offset(T, d, ff, E, k, 0, 0, dtype, which);
}

size_t moe_forward_ex_workspace_offset(int T, int d, int ff, int E, int k, int S, int F, int dtype, int which) {
    if (check_sizes(T, d, ff, E, k, dtype, true) != MOE_OK || check_shared(T, k, S) != MOE_OK ||
        check_reroute(k, E, F) != MOE_OK)
        return size_t(-1);
    const WsLayout L = ws_layout(T, d, ff, E, k, dtype, S, F);
    switch (which) {
        case MOE_WS_TOPK_IDX: return L.idx;
        case MOE_WS_TOPK_GATE: return L.gate;
        case MOE_WS_COUNTS: return L.counts;
        case MOE_WS_OFFSETS: return L.offsets;
        case MOE_WS_PERM: return L.perm;
        case MOE_WS_SLOT_OF: return L.slot_of;
        case MOE_WS_ROW_GATE: return L.row_gate;
        case MOE_WS_XP: return L.xp;
        case MOE_WS_H: return L.h;
        case MOE_WS_YP: return L.yp;
        case MOE_WS_FALLBACK_IDX: return L.fb_idx;
        case MOE_WS_FALLBACK_GATE: return L.fb_gate;
        default: return size_t(-1);
    }
}

size_t moe_dispatch_workspace_size(int T, int k, int E) {
    if (T < 0 || k < 1 || E < 1 || E > MOE_MAX_EXPERTS || static_cast<long long>(T) * k >= (1ll << 31)) return 0;
    return dispatch_ws_bytes(T * k, E);
}

int moe_router_topk(const void* x, const void* w_router, const float* logit_bias, int T, int d, int E, int k,
                    int dtype, int32_t* topk_idx, float* topk_gate, float* prob_sum, void* stream) {
    TraceRange trace_("moe_router_topk");
    int rc = check_sizes(T, d, 8, E, k, dtype, false);
    if (rc != MOE_OK) return rc;
    if (T == 0) {
        if (prob_sum != nullptr &&
            cudaMemsetAsync(prob_sum, 0, size_t(E) * 4, static_cast<cudaStream_t>(stream)) != cudaSuccess)
            return MOE_ERR_CUDA;
        return MOE_OK;
    }
    if (!x || !w_router || !topk_idx || !topk_gate) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(w_router)) return MOE_ERR_INVALID_ARG;
    RouterOut o{topk_idx, topk_gate, prob_sum, nullptr, nullptr, 0, nullptr, nullptr};
    return run_router(x, w_router, logit_bias, T, d, E, k, dtype, o, static_cast<cudaStream_t>(stream));
}

int moe_dispatch(const int32_t* topk_idx, const float* topk_gate, int T, int k, int E, int capacity,
                 int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* slot_of, uint8_t* drop_mask,
                 float* row_gate, const void* x, void* xp, int d, int dtype, void* ws, size_t ws_bytes,
                 void* stream) {
    TraceRange trace_("moe_dispatch");
    const bool want_rows = (x != nullptr || xp != nullptr);
    const int rc = want_rows ? check_sizes(T, d, 8, E, k, dtype, false) : check_sizes(T, 8, 8, E, k, MOE_F32, false);
    if (rc != MOE_OK) return rc;
    if (!counts || !offsets) return MOE_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (T == 0) {
        // no assignments: counts = 0, offsets = 0; the other pointers may be NULL
        if (cudaMemsetAsync(counts, 0, size_t(E) * 4, s) != cudaSuccess) return MOE_ERR_CUDA;
        if (cudaMemsetAsync(offsets, 0, size_t(E + 1) * 4, s) != cudaSuccess) return MOE_ERR_CUDA;
        return MOE_OK;
    }
    if (want_rows && (!x || !xp || !aligned16(x) || !aligned16(xp))) return MOE_ERR_INVALID_ARG;
    if (row_gate != nullptr && topk_gate == nullptr) return MOE_ERR_INVALID_ARG;
    if (!topk_idx || !perm || !slot_of) return MOE_ERR_INVALID_ARG;
    if (ws == nullptr || ws_bytes < dispatch_ws_bytes(T * k, E)) return MOE_ERR_WORKSPACE;
    return run_dispatch(topk_idx, topk_gate, T, k, E, capacity, counts, offsets, perm, slot_of, drop_mask, row_gate,
                        x, xp, d, dtype, ws, s);
}

int moe_dispatch_noalloc(const int32_t* topk_idx, const float* topk_gate, int T, int k, int E, int capacity,
                         int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* slot_of, uint8_t* drop_mask,
                         float* row_gate, const void* x, void* xp, int d, int dtype, void* stream) {
    TraceRange trace_("moe_dispatch_noalloc");
    const bool want_rows = (x != nullptr || xp != nullptr);
    const int rc = want_rows ? check_sizes(T, d, 8, E, k, dtype, false) : check_sizes(T, 8, 8, E, k, MOE_F32, false);
    if (rc != MOE_OK) return rc;
    if (static_cast<long long>(T) * k > MOE_NOALLOC_MAX_ASSIGNMENTS) {
        std::fprintf(stderr, "libmoe: moe_dispatch_noalloc: T*k = %lld exceeds the fixed scratch limit of %d "
                             "assignments; use moe_dispatch with a workspace\n",
                     static_cast<long long>(T) * k, MOE_NOALLOC_MAX_ASSIGNMENTS);
        return MOE_ERR_WORKSPACE;
    }
    if (!counts || !offsets) return MOE_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (T == 0) {
        if (cudaMemsetAsync(counts, 0, size_t(E) * 4, s) != cudaSuccess) return MOE_ERR_CUDA;
        if (cudaMemsetAsync(offsets, 0, size_t(E + 1) * 4, s) != cudaSuccess) return MOE_ERR_CUDA;
        return MOE_OK;
    }
    if (want_rows && (!x || !xp || !aligned16(x) || !aligned16(xp))) return MOE_ERR_INVALID_ARG;
    if (row_gate != nullptr && topk_gate == nullptr) return MOE_ERR_INVALID_ARG;
    if (!topk_idx || !perm || !slot_of) return MOE_ERR_INVALID_ARG;
    void* scratch = nullptr;
    const int src = noalloc_scratch(&scratch);
    if (src != MOE_OK) return src;
    // every histogram and base entry the kernels read is written earlier in
    // the same call, so nothing in the scratch needs clearing
    return run_dispatch(topk_idx, topk_gate, T, k, E, capacity, counts, offsets, perm, slot_of, drop_mask, row_gate,
                        x, xp, d, dtype, scratch, s);
}

// step-level rerouting dispatch: chunks of kRerouteChunk tokens
constexpr int kRerouteChunk = 128;

struct RerouteStepWs {
    size_t idx, gate, fb_idx, fb_gate, hist, base, reroute, total;
};

RerouteStepWs reroute_step_layout(int T, int k, int F, int E) {
    RerouteStepWs L{};
    const int nchunk = std::max(1, ceil_div(T, kRerouteChunk));
    size_t o = 0;
    auto take = [&](size_t bytes) {
        const size_t r = o;
        o += align256(std::max<size_t>(bytes, 1));
        return r;
    };
    L.idx = take(size_t(T) * k * 4);
    L.gate = take(size_t(T) * k * 4);
    L.fb_idx = take(size_t(T) * F * 4);
    L.fb_gate = take(size_t(T) * F * 4);
    L.hist = take(size_t(nchunk) * E * 4);
    L.base = take(size_t(nchunk) * E * 4);
    L.reroute = take(F > 0 ? reroute_ws_bytes(T, k, E, F, nchunk) : 0);
    L.total = o;
    return L;
}

size_t moe_dispatch_reroute_workspace_size(int T, int k, int F, int E) {
    if (T < 0 || k < 1 || E < 1 || E > MOE_MAX_EXPERTS || check_reroute(k, E, F) != MOE_OK ||
        static_cast<long long>(T) * (k + F) >= (1ll << 31))
        return 0;
    return reroute_step_layout(T, k, F, E).total;
}

int moe_dispatch_reroute(const int32_t* ranked_idx, const float* ranked_gate, int T, int k, int F, int E,
                         int capacity, int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* slot_of,
                         uint8_t* drop_mask, float* row_gate, const void* x, void* xp, int d, int dtype, void* ws,
                         size_t ws_bytes, void* stream) {
    TraceRange trace_("moe_dispatch_reroute");
    const bool want_rows = (x != nullptr || xp != nullptr);
    int rc = want_rows ? check_sizes(T, d, 8, E, k, dtype, false) : check_sizes(T, 8, 8, E, k, MOE_F32, false);
    if (rc != MOE_OK) return rc;
    if ((rc = check_reroute(k, E, F)) != MOE_OK) return rc;
    if (static_cast<long long>(T) * (k + F) >= (1ll << 31)) return MOE_ERR_UNSUPPORTED;
    if (!counts || !offsets) return MOE_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (T == 0) {
        if (cudaMemsetAsync(counts, 0, size_t(E) * 4, s) != cudaSuccess) return MOE_ERR_CUDA;
        if (cudaMemsetAsync(offsets, 0, size_t(E + 1) * 4, s) != cudaSuccess) return MOE_ERR_CUDA;
        return MOE_OK;
    }
    if (want_rows && (!x || !xp || !aligned16(x) || !aligned16(xp))) return MOE_ERR_INVALID_ARG;
    if (row_gate != nullptr && ranked_gate == nullptr) return MOE_ERR_INVALID_ARG;
    if (!ranked_idx || !perm || !slot_of) return MOE_ERR_INVALID_ARG;
    const RerouteStepWs L = reroute_step_layout(T, k, F, E);
    if (ws == nullptr || ws_bytes < L.total || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0)
        return MOE_ERR_WORKSPACE;
    uint8_t* w = static_cast<uint8_t*>(ws);
    int32_t* idx = reinterpret_cast<int32_t*>(w + L.idx);
    float* gate = reinterpret_cast<float*>(w + L.gate);
    int32_t* fb_idx = reinterpret_cast<int32_t*>(w + L.fb_idx);
    float* fb_gate = reinterpret_cast<float*>(w + L.fb_gate);
    int32_t* hist = reinterpret_cast<int32_t*>(w + L.hist);
    int32_t* base = reinterpret_cast<int32_t*>(w + L.base);
    const int nchunk = ceil_div(T, kRerouteChunk);
    {
        Launch Lk(MOE_KERNEL_COUNT, s);
        cudaError_t launch_err;
        launch_err = launch_pdl(reroute_split_kernel, dim3(nchunk), dim3(kFwdThreads), 0, s, ranked_idx, ranked_gate,
                                T, k, F, E, kRerouteChunk, idx, gate, fb_idx, fb_gate, hist);
        if ((rc = Lk.finish(launch_err)) != MOE_OK) return rc;
    }
    // without x the permute kernels gather nothing (zero row bytes)
    const int dd = want_rows ? d : 0;
    if (F > 0 && capacity >= 0)
        return run_reroute_dispatch(idx, gate, fb_idx, fb_gate, T, k, E, capacity, F, kRerouteChunk, hist, nullptr,
                                    base, counts, offsets, perm, slot_of, drop_mask, row_gate, nullptr, x, xp, dd,
                                    dtype, nullptr, carve_reroute_ws(w + L.reroute, T, k, E, F, nchunk), s);
    return run_forward_dispatch(idx, gate, T, k, E, capacity, kRerouteChunk, hist, nullptr, base, counts, offsets,
                                perm, slot_of, drop_mask, row_gate, nullptr, x, xp, dd, dtype, nullptr, s);
}

int moe_grouped_ffn(const void* xp, const int32_t* offsets, int max_rows, int E, int d, int ff, const void* w1,
                    const void* b1, const void* w2, const void* b2, const float* row_gate, void* h, void* yp,
                    int dtype, void* stream) {
    TraceRange trace_("moe_grouped_ffn");
    const int rc = check_sizes(max_rows, d, ff, E, 1, dtype, true);
    if (rc != MOE_OK) return rc;
    if (max_rows == 0) return MOE_OK;
    if (!xp || !offsets || !w1 || !b1 || !w2 || !b2 || !h || !yp) return MOE_ERR_INVALID_ARG;
    if (!aligned16(xp) || !aligned16(w1) || !aligned16(b1) || !aligned16(w2) || !aligned16(b2) || !aligned16(h) ||
        !aligned16(yp))
        return MOE_ERR_INVALID_ARG;
    return run_ffn(xp, offsets, max_rows, E, d, ff, w1, b1, w2, b2, row_gate, h, yp, dtype, nullptr,
                   SharedExperts{}, false, static_cast<cudaStream_t>(stream));
}

int moe_shared_ffn(const void* x, int T, int d, int ff, int S, const void* w1s, const void* b1s, const void* w2s,
                   const void* b2s, void* h, void* ys, int dtype, void* stream) {
    TraceRange trace_("moe_shared_ffn");
    int rc = check_sizes(T, d, ff, 1, 1, dtype, true);
    if (rc != MOE_OK) return rc;
    if ((rc = check_shared(T, 0, S)) != MOE_OK) return rc;
    if (T == 0 || S == 0) return MOE_OK;
    if (!x || !w1s || !b1s || !w2s || !b2s || !h || !ys) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(w1s) || !aligned16(b1s) || !aligned16(w2s) || !aligned16(b2s) ||
        !aligned16(h) || !aligned16(ys))
        return MOE_ERR_INVALID_ARG;
    SharedExperts se;
    se.S = S;
    se.T = T;
    se.x = x;
    se.w1 = w1s;
    se.b1 = b1s;
    se.w2 = w2s;
    se.b2 = b2s;
    return run_ffn(nullptr, nullptr, 0, 0, d, ff, nullptr, nullptr, nullptr, nullptr, nullptr, h, ys, dtype,
                   nullptr, se, false, static_cast<cudaStream_t>(stream));
}

int moe_combine(const void* yp, const int32_t* slot_of, const float* topk_gate, int T, int k, int d, int dtype,
                void* out, void* stream) {
    TraceRange trace_("moe_combine");
    const int rc = check_sizes(T, d, 8, k, k, dtype, false);
    if (rc != MOE_OK) return rc;
    if (T == 0) return MOE_OK;
    if (!yp || !slot_of || !out) return MOE_ERR_INVALID_ARG;
    if (!aligned16(yp) || !aligned16(out)) return MOE_ERR_INVALID_ARG;
    return run_combine(yp, slot_of, topk_gate, T, k, d, dtype, out, nullptr, 0, static_cast<cudaStream_t>(stream));
}

int moe_combine_shared(const void* yp, const int32_t* slot_of, const float* topk_gate, const void* ys, int S, int T,
                       int k, int d, int dtype, void* out, void* stream) {
    TraceRange trace_("moe_combine_shared");
    int rc = check_sizes(T, d, 8, k, k, dtype, false);
    if (rc != MOE_OK) return rc;
    if ((rc = check_shared(T, k, S)) != MOE_OK) return rc;
    if (T == 0) return MOE_OK;
    if (!yp || !slot_of || !out || (S > 0 && !ys)) return MOE_ERR_INVALID_ARG;
    if (!aligned16(yp) || !aligned16(out) || (S > 0 && !aligned16(ys))) return MOE_ERR_INVALID_ARG;
    return run_combine(yp, slot_of, topk_gate, T, k, d, dtype, out, ys, S, static_cast<cudaStream_t>(stream));
}

int moe_layer_stats(const int32_t* counts, const int32_t* offsets, const float* prob_sum, int T, int k, int E,
                    moe_stats* stats, void* stream) {
    TraceRange trace_("moe_layer_stats");
    const int rc = check_sizes(T, 8, 8, E, k, MOE_F32, false);
    if (rc != MOE_OK) return rc;
    if (T == 0) return MOE_ERR_INVALID_ARG;   // the statistics divide by T
    if (!counts || !offsets || !prob_sum || !stats) return MOE_ERR_INVALID_ARG;
    return run_stats(counts, offsets, prob_sum, T, k, E, stats, static_cast<cudaStream_t>(stream));
}

int moe_forward(const void* x, const void* w_router, const float* logit_bias, const void* w1, const void* b1,
                const void* w2, const void* b2, int T, int d, int ff, int E, int k, int capacity, int dtype,
                void* out, moe_stats* stats, int32_t* topk_idx_out, float* topk_gate_out, void* ws,
                size_t ws_bytes, void* stream) {
    TraceRange trace_("moe_forward");
    return moe_forward_ex(x, w_router, logit_bias, w1, b1, w2, b2, 0, nullptr, nullptr, nullptr, nullptr, 0, T, d,
                          ff, E, k, capacity, dtype, out, stats, topk_idx_out, topk_gate_out, ws, ws_bytes, stream);
}

int moe_forward_ex(const void* x, const void* w_router, const float* logit_bias, const void* w1, const void* b1,
                   const void* w2, const void* b2, int S, const void* w1s, const void* b1s, const void* w2s,
                   const void* b2s, int reroute_rounds, int T, int d, int ff, int E, int k, int capacity, int dtype,
                   void* out, moe_stats* stats, int32_t* topk_idx_out, float* topk_gate_out, void* ws,
                   size_t ws_bytes, void* stream) {
    TraceRange trace_("moe_forward_ex");
    int rc = check_sizes(T, d, ff, E, k, dtype, true);
    if (rc != MOE_OK) return rc;
    if ((rc = check_shared(T, k, S)) != MOE_OK) return rc;
    if ((rc = check_reroute(k, E, reroute_rounds)) != MOE_OK) return rc;
    if (T == 0) return MOE_OK;
    if (!x || !w_router || !w1 || !b1 || !w2 || !b2 || !out) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(w_router) || !aligned16(w1) || !aligned16(b1) || !aligned16(w2) ||
        !aligned16(b2) || !aligned16(out))
        return MOE_ERR_INVALID_ARG;
    if (S > 0 && (!w1s || !b1s || !w2s || !b2s || !aligned16(w1s) || !aligned16(b1s) || !aligned16(w2s) ||
                  !aligned16(b2s)))
        return MOE_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(T, d, ff, E, k, dtype, S, reroute_rounds);
    if (ws == nullptr || ws_bytes < L.total || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0)
        return MOE_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t* w = static_cast<uint8_t*>(ws);
    int32_t* idx = topk_idx_out ? topk_idx_out : reinterpret_cast<int32_t*>(w + L.idx);
    float* gate = topk_gate_out ? topk_gate_out : reinterpret_cast<float*>(w + L.gate);
    int32_t* counts = reinterpret_cast<int32_t*>(w + L.counts);
    int32_t* offsets = reinterpret_cast<int32_t*>(w + L.offsets);
    int32_t* perm = reinterpret_cast<int32_t*>(w + L.perm);
    int32_t* slot_of = reinterpret_cast<int32_t*>(w + L.slot_of);
    float* row_gate = reinterpret_cast<float*>(w + L.row_gate);
    int32_t* fhist = reinterpret_cast<int32_t*>(w + L.fhist);
    int32_t* fbase = reinterpret_cast<int32_t*>(w + L.fbase);
    float* fpsum = stats ? reinterpret_cast<float*>(w + L.fpsum) : nullptr;   // only the statistics need it
    int32_t* fb_idx = reinterpret_cast<int32_t*>(w + L.fb_idx);
    float* fb_gate = reinterpret_cast<float*>(w + L.fb_gate);
    void* xp = w + L.xp;
    void* h = w + L.h;
    void* yp = w + L.yp;
    const int A = T * k;
    const int chunk_tokens = router_chunk_tokens(dtype);
    // rerouting only matters when a capacity can drop assignments
    const int F = capacity >= 0 ? reroute_rounds : 0;
    // top-1 without shared experts: every token has one contribution, so fc2
    // writes the output row of its token directly (rows of dropped tokens
    // are zeroed by the dispatch) and no combine runs
    const bool direct = (k == 1 && S == 0);
    SharedExperts se;
    se.S = S;
    se.T = T;
    se.x = x;
    se.w1 = w1s;
    se.b1 = b1s;
    se.w2 = w2s;
    se.b2 = b2s;

    RouterOut ro{idx, gate, nullptr, fpsum, fhist, F, fb_idx, fb_gate};
    if ((rc = run_router(x, w_router, logit_bias, T, d, E, k, dtype, ro, s)) != MOE_OK) return rc;
    if (F > 0)
        rc = run_reroute_dispatch(idx, gate, fb_idx, fb_gate, T, k, E, capacity, F, chunk_tokens, fhist, fpsum,
                                  fbase, counts, offsets, perm, slot_of, nullptr, row_gate, stats, x, xp, d, dtype,
                                  direct ? out : nullptr,
                                  carve_reroute_ws(w + L.reroute, T, k, E, F, ceil_div(T, chunk_tokens)), s);
    else
        rc = run_forward_dispatch(idx, gate, T, k, E, capacity, chunk_tokens, fhist, fpsum, fbase, counts, offsets,
                                  perm, slot_of, nullptr, row_gate, stats, x, xp, d, dtype, direct ? out : nullptr,
                                  s);
    if (rc != MOE_OK) return rc;
    // CTA pairs once the routed experts average at least 384 rows (256-row
    // tiles then waste little on padding) or env MOE_PAIR_TILES forces it
    const bool use_pairs = pair_tiles_enabled(static_cast<long long>(A) >= 384ll * E);
    const bool fc1_pairs = fc1_pair_tiles_enabled(false);
    if ((rc = run_ffn(xp, offsets, A, E, d, ff, w1, b1, w2, b2, row_gate, h, direct ? out : yp, dtype,
                      direct ? perm : nullptr, se, use_pairs, s, fc1_pairs)) != MOE_OK)
        return rc;
    if (!direct) {
        const void* ys = static_cast<const uint8_t*>(yp) + size_t(A) * d * elem_bytes(dtype);
        if ((rc = run_combine(yp, slot_of, nullptr, T, k, d, dtype, out, ys, S, s)) != MOE_OK) return rc;
    }
    return MOE_OK;
}

int moe_get_error(void* stream) {
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return MOE_ERR_CUDA;
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_error_word, sizeof(int)) != cudaSuccess) return MOE_ERR_CUDA;
    const int zero = 0;
    if (v != 0 && cudaMemcpyToSymbol(g_error_word, &zero, sizeof(int)) != cudaSuccess) return MOE_ERR_CUDA;
    return v;
}

int moe_debug_gelu(const float* x, float* y, int n, int variant, void* stream) {
    if (n < 0 || variant < 0 || variant > 2) return MOE_ERR_INVALID_ARG;
    if (n == 0) return MOE_OK;
    if (!x || !y) return MOE_ERR_INVALID_ARG;
    if (variant == 2)
        gelu2_probe_kernel<<<std::min(ceil_div(n, 512), 1024), 256, 0, static_cast<cudaStream_t>(stream)>>>(x, y, n);
    else
        gelu_probe_kernel<<<std::min(ceil_div(n, 256), 1024), 256, 0, static_cast<cudaStream_t>(stream)>>>(x, y, n,
                                                                                                         variant);
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

int moe_debug_wait_timeout(int64_t limit_ns, void* stream) {
    if (limit_ns <= 0 || static_cast<uint64_t>(limit_ns) > kWaitLimitNs) return MOE_ERR_INVALID_ARG;
    wait_timeout_probe_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(uint64_t(limit_ns));
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

uint64_t moe_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int moe_timing_enable(int enable) {
    std::lock_guard<std::mutex> lk(g_timing.mu);
    if (enable) {
        while (g_timing.free_events.size() + 2 * g_timing.pending.size() < size_t(kEventPool)) {
            cudaEvent_t e;
            if (cudaEventCreate(&e) != cudaSuccess) return MOE_ERR_CUDA;
            g_timing.free_events.push_back(e);
        }
    }
    g_timing.enabled = enable != 0;
    return MOE_OK;
}

int moe_ffn_clock_enable(int enable) {
    const int on = enable ? 1 : 0;
    if (on) {
        // a fresh record: launches that ran before this call leave no trace
        void* rec = nullptr;
        if (cudaGetSymbolAddress(&rec, g_ffn_clock) != cudaSuccess) return MOE_ERR_CUDA;
        if (cudaMemset(rec, 0, sizeof(g_ffn_clock)) != cudaSuccess) return MOE_ERR_CUDA;
    }
    if (cudaMemcpyToSymbol(g_ffn_clock_on, &on, sizeof(on)) != cudaSuccess) return MOE_ERR_CUDA;
    return cudaDeviceSynchronize() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

int moe_ffn_clock_read(double* sm_mhz, double* span_us) {
    if (cudaDeviceSynchronize() != cudaSuccess) return MOE_ERR_CUDA;
    std::vector<unsigned long long> rec(size_t(2) * kClockCtas * 4);
    if (cudaMemcpyFromSymbol(rec.data(), g_ffn_clock, sizeof(g_ffn_clock)) != cudaSuccess) return MOE_ERR_CUDA;
    for (int m = 0; m < 2; ++m) {
        std::vector<double> mhz;
        unsigned long long t_lo = ~0ull, t_hi = 0;
        for (int c = 0; c < kClockCtas; ++c) {
            const unsigned long long* r = rec.data() + (size_t(m) * kClockCtas + c) * 4;
            if (r[1] == 0 || r[3] <= r[1]) continue;   // no launch, or one still running
            mhz.push_back(double(r[2] - r[0]) / double(r[3] - r[1]) * 1e3);
            t_lo = std::min(t_lo, r[1]);
            t_hi = std::max(t_hi, r[3]);
        }
        double med = 0.0;
        if (!mhz.empty()) {
            std::sort(mhz.begin(), mhz.end());
            const size_t n = mhz.size();
            med = (n & 1) ? mhz[n / 2] : 0.5 * (mhz[n / 2 - 1] + mhz[n / 2]);
        }
        if (sm_mhz) sm_mhz[m] = med;
        if (span_us) span_us[m] = mhz.empty() ? 0.0 : double(t_hi - t_lo) * 1e-3;
    }
    return MOE_OK;
}

int moe_trace_enable(int enable) {
    const int prev = trace_on() ? 1 : 0;
    g_trace.store(enable ? 1 : 0, std::memory_order_relaxed);
    return prev;
}

int moe_trace_enabled(void) { return trace_on() ? 1 : 0; }

int moe_timing_read(double* ms_per_kernel, int64_t* launches_per_kernel) {
    std::lock_guard<std::mutex> lk(g_timing.mu);
    harvest_locked(g_timing.pending.size());
    for (int i = 0; i < MOE_NUM_KERNELS; ++i) {
        if (ms_per_kernel) ms_per_kernel[i] = g_timing.ms[i];
        if (launches_per_kernel) launches_per_kernel[i] = g_timing.launches[i];
        g_timing.ms[i] = 0.0;
        g_timing.launches[i] = 0;
    }
    return MOE_OK;
}

}  // extern "C"

#include "pipeline.cuh"
