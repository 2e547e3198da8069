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
// It runs the same tensor-core split-KV decode kernel and merge kernel as pa_forward; only
// where their scratch lives differs.
#include <algorithm>
#include <mutex>

#include "pa_internal.h"

namespace pa {
namespace {

// The fixed scratch array. Every GPU that loads this library holds it until the process
// exits. Layout: [work units][merge units][float32 parts: outputs, then logsumexps].
constexpr size_t kStaticBytes = (size_t)PA_STATIC_WORKSPACE_BYTES;
constexpr int kMaxUnits = 32768;        // 1 MiB of KvUnit
constexpr int kMaxMergeUnits = 32768;   // 512 KiB of CombineUnit
constexpr size_t kUnitsOff = 0;
constexpr size_t kMergeOff = kUnitsOff + sizeof(KvUnit) * kMaxUnits;
constexpr size_t kPartsOff = kMergeOff + sizeof(CombineUnit) * kMaxMergeUnits;
static_assert(kPartsOff % 256 == 0, "parts must start 256-byte aligned");
static_assert(kPartsOff < kStaticBytes, "scratch too small for its unit lists");

static __device__ __align__(256) unsigned char g_static_scratch[kStaticBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;                          // one call at a time uses the host staging lists
void* g_dev_ptr[kMaxDevices] = {};        // address of g_static_scratch on each device
KvUnit g_units[kMaxUnits];                // host staging of the work list
CombineUnit g_merge[kMaxMergeUnits];      // host staging of the merge list

// The device address of the scratch array on the current device (looked up once per device;
// the symbol's host-side name is not a device address).
pa_status scratch_on_device(int dev, void** out) {
    if (dev < 0 || dev >= kMaxDevices)
        return set_error(PA_ERR_UNSUPPORTED, "device ordinal %d is beyond this entry point's table", dev);
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

    std::lock_guard<std::mutex> lock(g_mu);
    void* base = nullptr;
    st = scratch_on_device(pv.device, &base);
    if (st != PA_OK) return st;

    // Keys each sequence's queries can see, and the automatic split size of pa_forward.
    int64_t total = 0;
    for (int32_t s = 0; s < pv.S; ++s) {
        const SeqInfo& si = pv.host_seqs[s];
        if (si.n == 0) continue;
        if ((int64_t)si.n * G > kDecodeMaxRows)
            return set_error(PA_ERR_UNSUPPORTED,
                             "sequence %d has %d query rows per KV head; the fixed-workspace decode takes at most %d",
                             s, si.n * G, kDecodeMaxRows);
        const int64_t p_first = (int64_t)si.L - si.n, p_last = (int64_t)si.L - 1;
        const int64_t lo = window > 0 ? std::max<int64_t>(0, p_first - window + 1) : 0;
        const int64_t hi = causal ? std::min<int64_t>(si.L, p_last + 1) : si.L;
        total += std::max<int64_t>(0, hi - lo) * num_kv_heads;
    }
    int64_t chunk;
    if (kv_chunk > 0) chunk = kv_chunk;
    else if (kv_chunk < 0) chunk = INT32_MAX;
    else {
        const int64_t target = (int64_t)pv.num_sms * 8;
        chunk = std::max<int64_t>(((total + target - 1) / target + 63) / 64 * 64, 256);
    }

    // Work list and merge list, straight into the host staging arrays.
    int32_t nu = 0, nm = 0;
    int64_t slots = 0;
    int32_t rows_max = 0;
    for (int32_t s = 0; s < pv.S; ++s) {
        const SeqInfo& si = pv.host_seqs[s];
        if (si.n == 0) continue;
        const int64_t p_first = (int64_t)si.L - si.n, p_last = (int64_t)si.L - 1;
        const int64_t lo = window > 0 ? std::max<int64_t>(0, p_first - window + 1) : 0;
        const int64_t hi = std::max<int64_t>(lo, causal ? std::min<int64_t>(si.L, p_last + 1) : si.L);
        const int64_t len = hi - lo;
        const int32_t nsplit = len <= 0 ? 1 : (int32_t)((len + chunk - 1) / chunk);
        if (nu + nsplit > kMaxUnits || (nsplit > 1 && nm + si.n > kMaxMergeUnits))
            return set_error(PA_ERR_BOUNDS, "batch needs more work units than the fixed workspace holds (%d)", kMaxUnits);
        const int32_t part_base = nsplit > 1 ? (int32_t)slots : -1;
        if (nsplit > 1) {
            for (int32_t j = 0; j < si.n; ++j) g_merge[nm++] = {si.q_start + j, part_base + j * nsplit, nsplit, 0};
            slots += (int64_t)si.n * nsplit;
        }
        for (int32_t i = 0; i < nsplit; ++i) {
            KvUnit& u = g_units[nu++];
            u.seq = s;
            u.t0 = (int32_t)std::min<int64_t>(hi, lo + i * chunk);
            u.t1 = (int32_t)std::min<int64_t>(hi, lo + (i + 1) * chunk);
            u.split = i;
            u.nsplit = nsplit;
            u.part_base = part_base;
            u.j0 = 0;
            u.j1 = si.n;
        }
        rows_max = std::max<int32_t>(rows_max, si.n * G);
    }
    const size_t part_bytes = (size_t)slots * num_q_heads * (v_head_dim + 1) * sizeof(float);
    if (part_bytes > kStaticBytes - kPartsOff)
        return set_error(PA_ERR_BOUNDS,
                         "split parts need %zu bytes but the fixed workspace holds %zu; pass a larger kv_chunk "
                         "(or -1) or use pa_forward",
                         part_bytes, (size_t)(kStaticBytes - kPartsOff));
    // Longest units first, in place (std::sort allocates nothing).
    std::sort(g_units, g_units + nu, [](const KvUnit& a, const KvUnit& b) {
        if (a.t1 - a.t0 != b.t1 - b.t0) return a.t1 - a.t0 > b.t1 - b.t0;
        if (a.seq != b.seq) return a.seq < b.seq;
        return a.split < b.split;
    });

    cudaStream_t cs = (cudaStream_t)stream;
    unsigned char* dev = static_cast<unsigned char*>(base);
    // Pageable source: each copy returns once the staging arrays have been read, so the next
    // call may refill them. The unit lists are rewritten in full on every call; the parts need
    // no clearing (every part the merge reads is written by this call first).
    cudaError_t e = cudaMemcpyAsync(dev + kUnitsOff, g_units, sizeof(KvUnit) * nu, cudaMemcpyHostToDevice, cs);
    if (e == cudaSuccess && nm > 0)
        e = cudaMemcpyAsync(dev + kMergeOff, g_merge, sizeof(CombineUnit) * nm, cudaMemcpyHostToDevice, cs);
    if (e != cudaSuccess) return set_error(PA_ERR_CUDA, "work list copy failed: %s", cudaGetErrorString(e));

    AttnParams p{};
    p.q = q; p.k = k_cache; p.v = v_cache;
    p.out = out; p.lse = lse;
    p.ws_o = reinterpret_cast<float*>(dev + kPartsOff);
    p.ws_lse = p.ws_o + (size_t)slots * num_q_heads * v_head_dim;
    p.seqs = pv.d_seqs;
    p.block_tables = pv.d_bt;
    p.units = reinterpret_cast<const KvUnit*>(dev + kUnitsOff);
    p.num_units = nu;
    p.cunits = reinterpret_cast<const CombineUnit*>(dev + kMergeOff);
    p.num_cunits = nm;
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
