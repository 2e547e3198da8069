// pa_forward_static_workspace: split-KV paged decode that allocates no memory.
//
// Some callers cannot allocate device memory while they run attention: a serving loop that
// must not stall on the allocator in the middle of a decode step, a process that runs under
// a fixed, pre-reserved memory budget, or an embedding runtime that does not let plugins call
// cudaMalloc at all. pa_forward may allocate (the split workspace grows on demand, and the
// first call with a new head configuration uploads its work list into fresh memory). This
// entry point instead keeps its work list and its float32 split parts in one fixed array in
// device global memory, defined below, so a call makes no allocation of any kind.
//
// The work list is not copied from the host: a one-CTA kernel writes it into the array from
// the plan's sequence table (already on the device), so the call issues no host-to-device copy
// and never waits on the stream. It then runs the same tensor-core split-KV decode kernel and
// merge kernel as pa_forward; only where their scratch lives, and the order of the work units
// (full-length parts of every sequence first, then each sequence's last, shorter part, where
// pa_forward sorts them longest first on the host), differ.
#include <algorithm>
#include <mutex>

#include "device_common.cuh"

namespace pa {
namespace {

// The fixed scratch array. Every GPU that loads this library holds it until the process
// exits. Layout: [work units][merge units][float32 parts: outputs, then logsumexps].
constexpr size_t kStaticBytes = (size_t)PA_STATIC_WORKSPACE_BYTES;
constexpr int kMaxUnits = 32768;        // 1 MiB of KvUnit
constexpr int kMaxMergeUnits = 16384;   // 256 KiB of CombineUnit
constexpr int kMaxParts = 1024;         // parts per sequence: the merge kernel's weight table
constexpr size_t kUnitsOff = 0;
constexpr size_t kMergeOff = kUnitsOff + sizeof(KvUnit) * kMaxUnits;
constexpr size_t kPartsOff = kMergeOff + sizeof(CombineUnit) * kMaxMergeUnits;
static_assert(kPartsOff % 256 == 0, "parts must start 256-byte aligned");
static_assert(kPartsOff < kStaticBytes, "scratch too small for its unit lists");

static __device__ __align__(256) unsigned char g_static_scratch[kStaticBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;                    // guards the address table
void* g_dev_ptr[kMaxDevices] = {};  // address of g_static_scratch on each device

// The device address of the scratch array on the current device (looked up once per device;
// the symbol's host-side name is not a device address).
pa_status scratch_on_device(int dev, void** out) {
    if (dev < 0 || dev >= kMaxDevices)
        return set_error(PA_ERR_UNSUPPORTED, "device ordinal %d is beyond this entry point's table", dev);
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_dev_ptr[dev]) {
        void* ptr = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&ptr, g_static_scratch);
        if (e != cudaSuccess || !ptr)
            return set_error(PA_ERR_CUDA, "cudaGetSymbolAddress of the fixed workspace failed: %s",
                             cudaGetErrorString(e));
        g_dev_ptr[dev] = ptr;
    }
    *out = g_dev_ptr[dev];
    return PA_OK;
}

// How one sequence's visible keys are cut into parts. The host (to check the limits and size
// the launches) and the list-building kernel (to write the units) both call this, on the same
// sequence table, so they agree on every count.
struct SeqSplit {
    int32_t lo, hi;  // keys [lo, hi) that some query of the sequence sees
    int32_t chunk;   // keys per part
    int32_t nsplit;  // parts (>= 1; a sequence without visible keys has one empty part)
};
__host__ __device__ __forceinline__ SeqSplit seq_split(const SeqInfo& si, int causal, int32_t window,
                                                       int64_t chunk) {
    const int64_t p_first = (int64_t)si.L - si.n, p_last = (int64_t)si.L - 1;
    const int64_t lo = window > 0 ? max64(0, p_first - window + 1) : 0;
    const int64_t hi = max64(lo, causal ? min64(si.L, p_last + 1) : si.L);
    const int64_t len = hi - lo;
    int64_t c = chunk;
    int64_t ns = len <= 0 ? 1 : (len + c - 1) / c;
    if (ns > kMaxParts) {  // pa_forward's rule: longer parts rather than more of them
        c = (len + kMaxParts - 1) / kMaxParts;
        ns = (len + c - 1) / c;
    }
    return SeqSplit{(int32_t)lo, (int32_t)hi, (int32_t)min64(c, INT32_MAX), (int32_t)ns};
}

// Exclusive prefix sums over the CTA of four counters per thread; `total` gets the CTA's sums.
__device__ __forceinline__ int4 block_exclusive_scan(int4 v, int4* total) {
    __shared__ int4 warp_sums[32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = (blockDim.x + 31) >> 5;
    int4 inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int a = __shfl_up_sync(0xffffffffu, inc.x, o), b = __shfl_up_sync(0xffffffffu, inc.y, o);
        const int c = __shfl_up_sync(0xffffffffu, inc.z, o), d = __shfl_up_sync(0xffffffffu, inc.w, o);
        if (lane >= o) { inc.x += a; inc.y += b; inc.z += c; inc.w += d; }
    }
    if (lane == 31) warp_sums[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        int4 s = lane < nwarps ? warp_sums[lane] : make_int4(0, 0, 0, 0);
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int a = __shfl_up_sync(0xffffffffu, s.x, o), b = __shfl_up_sync(0xffffffffu, s.y, o);
            const int c = __shfl_up_sync(0xffffffffu, s.z, o), d = __shfl_up_sync(0xffffffffu, s.w, o);
            if (lane >= o) { s.x += a; s.y += b; s.z += c; s.w += d; }
        }
        if (lane < nwarps) warp_sums[lane] = s;  // inclusive sums of the warps
    }
    __syncthreads();
    const int4 before = warp > 0 ? warp_sums[warp - 1] : make_int4(0, 0, 0, 0);
    *total = warp_sums[nwarps - 1];
    __syncthreads();  // warp_sums is rewritten by the next call
    return make_int4(before.x + inc.x - v.x, before.y + inc.y - v.y, before.z + inc.z - v.z, before.w + inc.w - v.w);
}

constexpr int kListThreads = 1024;

// One CTA walks the sequences kListThreads at a time. Sequence s with n > 0 queries and
// nsplit parts contributes nsplit - 1 full-length units (placed first, in sequence order), its
// last unit (placed after all full-length ones), and, when split, one merge unit per query.
__global__ void __launch_bounds__(kListThreads) build_lists_kernel(const SeqInfo* seqs, int32_t S, int causal,
                                                                   int32_t window, int64_t chunk, int32_t n_full,
                                                                   KvUnit* units, CombineUnit* merge) {
    int4 carry = make_int4(0, 0, 0, 0);  // full units, last units, merge units, part slots so far
    for (int32_t base = 0; base < S; base += kListThreads) {
        const int32_t s = base + (int32_t)threadIdx.x;
        SeqInfo si{0, 0, 0, 0};
        SeqSplit sp{0, 0, 1, 1};
        int4 cnt = make_int4(0, 0, 0, 0);
        if (s < S) {
            si = seqs[s];
            if (si.n > 0) {
                sp = seq_split(si, causal, window, chunk);
                cnt = make_int4(sp.nsplit - 1, 1, sp.nsplit > 1 ? si.n : 0, sp.nsplit > 1 ? si.n * sp.nsplit : 0);
            }
        }
        int4 total;
        const int4 ex = block_exclusive_scan(cnt, &total);
        if (cnt.y) {
            const int32_t part_base = sp.nsplit > 1 ? carry.w + ex.w : -1;
            for (int32_t i = 0; i < sp.nsplit; ++i) {
                KvUnit u;
                u.seq = s;
                u.t0 = (int32_t)min64(sp.hi, (int64_t)sp.lo + (int64_t)i * sp.chunk);
                u.t1 = (int32_t)min64(sp.hi, (int64_t)sp.lo + (int64_t)(i + 1) * sp.chunk);
                u.split = i;
                u.nsplit = sp.nsplit;
                u.part_base = part_base;
                u.j0 = 0;
                u.j1 = si.n;
                units[i + 1 < sp.nsplit ? carry.x + ex.x + i : n_full + carry.y + ex.y] = u;
            }
            for (int32_t j = 0; j < cnt.z; ++j)
                merge[carry.z + ex.z + j] = CombineUnit{si.q_start + j, part_base + j * sp.nsplit, sp.nsplit, 0};
        }
        carry = make_int4(carry.x + total.x, carry.y + total.y, carry.z + total.z, carry.w + total.w);
    }
}

}  // namespace
}  // namespace pa

extern "C" pa_status pa_forward_static_workspace(pa_plan* plan, const void* q, const void* k_cache,
                                                 const void* v_cache, pa_dtype dtype, int32_t num_q_heads,
                                                 int32_t num_kv_heads, int32_t head_dim, int32_t v_head_dim,
                                                 float scale, int causal, int32_t window, int32_t kv_chunk,
                                                 void* out, float* lse, pa_stream stream) {
    using namespace pa;
    PlanView pv{};
    pa_status st = validated_gqa_view(plan, q, k_cache, v_cache, dtype, num_q_heads, num_kv_heads, head_dim,
                                      v_head_dim, scale, causal, window, out, lse, &pv);
    if (st != PA_OK) return st;
    if (kv_chunk < -1) return set_error(PA_ERR_INVALID_ARGUMENT, "kv_chunk must be -1, 0 or > 0");
    if (pv.Nq == 0) return clear_error();
    const int32_t G = num_q_heads / num_kv_heads;
    if (dtype == PA_F32 || head_dim != v_head_dim || (head_dim != 64 && head_dim != 128))
        return set_error(PA_ERR_UNSUPPORTED,
                         "the fixed-workspace decode takes bf16/fp16 with head_dim == v_head_dim in {64, 128}");

    // Keys each sequence's queries can see, and the automatic split size of pa_forward.
    int64_t total = 0;
    for (int32_t s = 0; s < pv.S; ++s) {
        const SeqInfo& si = pv.host_seqs[s];
        if (si.n == 0) continue;
        if ((int64_t)si.n * G > kDecodeMaxRows)
            return set_error(PA_ERR_UNSUPPORTED,
                             "sequence %d has %d query rows per KV head; the fixed-workspace decode takes at most %d",
                             s, si.n * G, kDecodeMaxRows);
        const SeqSplit sp = seq_split(si, causal, window, INT32_MAX);
        total += (int64_t)(sp.hi - sp.lo) * num_kv_heads;
    }
    int64_t chunk;
    if (kv_chunk > 0) chunk = kv_chunk;
    else if (kv_chunk < 0) chunk = INT32_MAX;
    else {
        const int64_t target = (int64_t)pv.num_sms * 8;
        chunk = std::max<int64_t>(((total + target - 1) / target + 63) / 64 * 64, 256);
    }

    // The counts the list-building kernel will produce, checked against the array's limits.
    int64_t nu = 0, n_full = 0, nm = 0, slots = 0;
    int32_t rows_max = 0;
    for (int32_t s = 0; s < pv.S; ++s) {
        const SeqInfo& si = pv.host_seqs[s];
        if (si.n == 0) continue;
        const SeqSplit sp = seq_split(si, causal, window, chunk);
        nu += sp.nsplit;
        n_full += sp.nsplit - 1;
        if (sp.nsplit > 1) {
            nm += si.n;
            slots += (int64_t)si.n * sp.nsplit;
        }
        rows_max = std::max<int32_t>(rows_max, si.n * G);
    }
    if (nu > kMaxUnits)
        return set_error(PA_ERR_BOUNDS,
                         "batch needs %lld work units but the fixed workspace holds %d; pass a larger kv_chunk "
                         "(or -1), use fewer sequences per call, or use pa_forward",
                         (long long)nu, kMaxUnits);
    if (nm > kMaxMergeUnits)
        return set_error(PA_ERR_BOUNDS,
                         "batch needs %lld merge units (split query rows) but the fixed workspace holds %d; pass a "
                         "larger kv_chunk (or -1) or use pa_forward",
                         (long long)nm, kMaxMergeUnits);
    const size_t part_bytes = (size_t)slots * num_q_heads * (v_head_dim + 1) * sizeof(float);
    if (part_bytes > kStaticBytes - kPartsOff)
        return set_error(PA_ERR_BOUNDS,
                         "split parts need %zu bytes but the fixed workspace holds %zu; pass a larger kv_chunk "
                         "(or -1) or use pa_forward",
                         part_bytes, (size_t)(kStaticBytes - kPartsOff));

    void* base = nullptr;
    st = scratch_on_device(pv.device, &base);
    if (st != PA_OK) return st;

    cudaStream_t cs = (cudaStream_t)stream;
    unsigned char* dev = static_cast<unsigned char*>(base);
    KvUnit* units = reinterpret_cast<KvUnit*>(dev + kUnitsOff);
    CombineUnit* merge = reinterpret_cast<CombineUnit*>(dev + kMergeOff);
    // The unit lists are rewritten in full on every call; the parts need no clearing (every part
    // the merge reads is written by this call first).
    build_lists_kernel<<<1, kListThreads, 0, cs>>>(pv.d_seqs, pv.S, causal, window, chunk, (int32_t)n_full, units,
                                                   merge);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return set_error(PA_ERR_CUDA, "work list kernel launch failed: %s", cudaGetErrorString(e));

    AttnParams p{};
    p.q = q; p.k = k_cache; p.v = v_cache;
    p.out = out; p.lse = lse;
    p.ws_o = reinterpret_cast<float*>(dev + kPartsOff);
    p.ws_lse = p.ws_o + (size_t)slots * num_q_heads * v_head_dim;
    p.seqs = pv.d_seqs;
    p.block_tables = pv.d_bt;
    p.units = units;
    p.num_units = (int32_t)nu;
    p.cunits = merge;
    p.num_cunits = (int32_t)nm;
    p.table_width = pv.table_width;
    p.page_size = pv.page_size;
    p.hq = num_q_heads; p.hkv = num_kv_heads; p.group = G;
    p.d = head_dim; p.dv = v_head_dim; p.pr = 0;
    p.scale = scale;
    p.scale_log2 = (float)((double)scale * 1.4426950408889634);
    p.causal = causal; p.window = window;
    p.num_queries = pv.Nq;
    p.num_pages = pv.num_pages;
    p.err = pv.d_err;
    if (nu > 0) {
        e = launch_decode_mma(p, dtype, rows_max, cs);
        if (e != cudaSuccess) return set_error(PA_ERR_CUDA, "decode kernel launch failed: %s", cudaGetErrorString(e));
    }
    if (nm > 0) {
        e = launch_combine(p, dtype, cs);
        if (e != cudaSuccess) return set_error(PA_ERR_CUDA, "merge kernel launch failed: %s", cudaGetErrorString(e));
    }
    return clear_error();
}
