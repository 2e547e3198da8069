// Host side of libpa.so: the C ABI, argument validation, the plan (schedule upload and
// split workspace) and kernel dispatch.
//
// Validation follows ruDNN's paged_attention/mod.rs (`check_tensor`, `bounded`,
// `execute_attention_into`): every argument is checked before anything is launched or
// allocated, and an empty batch returns success without a launch.
#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <deque>
#include <functional>
#include <memory>
#include <mutex>
#include <unordered_map>
#include <vector>

#include "pa_internal.h"

namespace {

thread_local char g_msg[512] = "";

pa_status fail(pa_status st, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_msg, sizeof g_msg, fmt, ap);
    va_end(ap);
    return st;
}

pa_status ok() {
    g_msg[0] = '\0';
    return PA_OK;
}

#define PA_CUDA_TRY(expr)                                                                    \
    do {                                                                                     \
        cudaError_t e_ = (expr);                                                             \
        if (e_ != cudaSuccess)                                                               \
            return fail(PA_ERR_CUDA, "%s failed: %s", #expr, cudaGetErrorString(e_));        \
    } while (0)

size_t dtype_size(pa_dtype dt) { return dt == PA_F32 ? 4 : 2; }

bool mul_ok(int64_t a, int64_t b, int64_t* r) { return !__builtin_mul_overflow(a, b, r); }

// Product of non-negative dims; false on overflow of int64.
bool product(std::initializer_list<int64_t> dims, int64_t* r) {
    int64_t acc = 1;
    for (int64_t d : dims) {
        if (d < 0 || !mul_ok(acc, d, &acc)) return false;
    }
    *r = acc;
    return true;
}

struct Range {
    uintptr_t lo, hi;  // [lo, hi)
};
bool overlap(Range a, Range b) { return a.lo < b.hi && b.lo < a.hi && a.hi > a.lo && b.hi > b.lo; }

constexpr int kMaxSplits = 1024;           // parts one sequence's keys may be cut into

// ---------------------------------------------------------------------------------------
// Host-to-device uploads through pinned staging
// ---------------------------------------------------------------------------------------
// A copy from pageable memory makes the driver stage it itself (synchronously, and it may wait
// for the stream); copies through page-locked slots are true asynchronous DMA. The slots are
// allocated once per process and shared by every plan; a slot is reused once the event recorded
// after its last copy has completed. Uploads larger than a slot go through several slots.
constexpr int kStageSlots = 16;
constexpr size_t kStageSlotBytes = 256 << 10;

struct Staging {
    std::mutex mu;
    char* slot[kStageSlots] = {};
    cudaEvent_t done[kStageSlots] = {};
    bool used[kStageSlots] = {};
    int next = 0;
};
constexpr int kStageDevices = 64;
Staging* staging(int dev) {  // one set of slots per device (events belong to a device)
    static std::mutex mu;
    static Staging* per_dev[kStageDevices] = {};  // never destroyed: outlive any plan released at exit
    if (dev < 0 || dev >= kStageDevices) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!per_dev[dev]) per_dev[dev] = new Staging();
    return per_dev[dev];
}

// Device memory of plans (metadata, work lists, workspaces) comes from a pool of the library's
// own per device that keeps freed memory cached (release threshold at its maximum), and the
// process's default pool is left as the caller configured it.
cudaError_t pool_malloc(void** ptr, size_t bytes, cudaStream_t st) {
    static std::mutex mu;
    static cudaMemPool_t pools[kStageDevices] = {};
    static bool tried[kStageDevices] = {};
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    cudaMemPool_t pool = nullptr;
    if (dev >= 0 && dev < kStageDevices) {
        std::lock_guard<std::mutex> lock(mu);
        if (!tried[dev]) {
            tried[dev] = true;
            cudaMemPoolProps props = {};
            props.allocType = cudaMemAllocationTypePinned;
            props.location.type = cudaMemLocationTypeDevice;
            props.location.id = dev;
            cudaMemPool_t pl = nullptr;
            if (cudaMemPoolCreate(&pl, &props) == cudaSuccess) {
                uint64_t keep = UINT64_MAX;
                cudaMemPoolSetAttribute(pl, cudaMemPoolAttrReleaseThreshold, &keep);
                pools[dev] = pl;
            }
        }
        pool = pools[dev];
    }
    if (!pool) return cudaMallocAsync(ptr, bytes, st);
    return cudaMallocFromPoolAsync(ptr, bytes, pool, st);
}

// Freed plan memory first waits in a per-device list, with an event recorded on the stream that
// freed it; an allocation takes the oldest listed block of a fitting size (at most twice the
// request) whose event has completed, so that a new plan per decode step reuses an earlier step's
// memory without a driver call. (Plans allocate on their upload stream and free on their call
// stream, so the pool can reuse such memory only through a cross-stream dependency or maps more;
// its allocations were measured at 3-52 us per plan.) The list keeps at most kRecycleBytes; older
// blocks go back to the pool, stream-ordered after their event. Calls on a capturing stream use
// the pool directly.
struct Recycled {
    void* p;
    size_t bytes;
    cudaEvent_t ev;
};
struct Recycler {
    std::mutex mu;
    std::unordered_map<void*, size_t> sizes;  // every block handed out by lib_malloc, rounded size
    std::deque<Recycled> list;                // freed blocks, oldest first
    size_t held = 0;
    std::vector<cudaEvent_t> spare;           // completed events, for reuse
};
constexpr size_t kRecycleBytes = size_t(256) << 20;
constexpr size_t kRecycleGrain = size_t(64) << 10;
Recycler* recycler(int dev) {
    static std::mutex mu;
    static Recycler* per_dev[kStageDevices] = {};  // never destroyed: outlive any plan released at exit
    if (dev < 0 || dev >= kStageDevices) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!per_dev[dev]) per_dev[dev] = new Recycler();
    return per_dev[dev];
}
bool capturing(cudaStream_t st) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    return cudaStreamIsCapturing(st, &cs) == cudaSuccess && cs != cudaStreamCaptureStatusNone;
}

cudaError_t lib_malloc(void** ptr, size_t bytes, cudaStream_t st) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    Recycler* R = capturing(st) ? nullptr : recycler(dev);
    if (!R) return pool_malloc(ptr, bytes, st);
    const size_t want = (std::max<size_t>(bytes, 1) + kRecycleGrain - 1) / kRecycleGrain * kRecycleGrain;
    std::lock_guard<std::mutex> lock(R->mu);
    for (auto it = R->list.begin(); it != R->list.end(); ++it) {
        if (it->bytes < want || it->bytes > 2 * want) continue;
        const cudaError_t q = cudaEventQuery(it->ev);
        if (q == cudaErrorNotReady) continue;  // its last user is still queued
        if (q != cudaSuccess) return q;
        *ptr = it->p;
        R->spare.push_back(it->ev);
        R->held -= it->bytes;
        R->list.erase(it);
        return cudaSuccess;
    }
    e = pool_malloc(ptr, want, st);
    if (e == cudaSuccess) R->sizes[*ptr] = want;
    return e;
}

// Release a block from lib_malloc after the work queued on `st` so far (device `dev`).
cudaError_t lib_free(void* p, int dev, cudaStream_t st) {
    if (!p) return cudaSuccess;
    Recycler* R = capturing(st) ? nullptr : recycler(dev);
    if (!R) return cudaFreeAsync(p, st);
    std::lock_guard<std::mutex> lock(R->mu);
    auto f = R->sizes.find(p);
    if (f == R->sizes.end()) return cudaFreeAsync(p, st);
    const size_t bytes = f->second;
    int cur = -1;
    cudaError_t e = cudaGetDevice(&cur);
    if (e != cudaSuccess) return e;
    if (cur != dev && (e = cudaSetDevice(dev)) != cudaSuccess) return e;
    cudaEvent_t ev = nullptr;
    if (!R->spare.empty()) {
        ev = R->spare.back();
        R->spare.pop_back();
    } else {
        e = cudaEventCreateWithFlags(&ev, cudaEventDisableTiming);
    }
    if (e == cudaSuccess) e = cudaEventRecord(ev, st);
    if (e == cudaSuccess) {
        R->list.push_back({p, bytes, ev});
        R->held += bytes;
        while (R->held > kRecycleBytes && e == cudaSuccess) {
            const Recycled old = R->list.front();
            R->list.pop_front();
            R->held -= old.bytes;
            R->sizes.erase(old.p);
            R->spare.push_back(old.ev);
            e = cudaStreamWaitEvent(st, old.ev, 0);
            if (e == cudaSuccess) e = cudaFreeAsync(old.p, st);
        }
    } else {
        if (ev) R->spare.push_back(ev);
        R->sizes.erase(f);
        e = cudaFreeAsync(p, st);
    }
    if (cur != dev) cudaSetDevice(cur);
    return e;
}

cudaError_t upload_slot(Staging& g, void* dst, const void* src, size_t bytes, cudaStream_t st) {
    std::lock_guard<std::mutex> lock(g.mu);
    const int i = g.next;
    g.next = (g.next + 1) % kStageSlots;
    cudaError_t e;
    if (!g.slot[i]) {
        if ((e = cudaMallocHost(reinterpret_cast<void**>(&g.slot[i]), kStageSlotBytes)) != cudaSuccess) {
            g.slot[i] = nullptr;
            return cudaMemcpyAsync(dst, src, bytes, cudaMemcpyHostToDevice, st);
        }
        if ((e = cudaEventCreateWithFlags(&g.done[i], cudaEventDisableTiming)) != cudaSuccess) return e;
    } else if (g.used[i] && (e = cudaEventSynchronize(g.done[i])) != cudaSuccess) {
        return e;  // the slot's previous copy has to finish before it is overwritten
    }
    std::memcpy(g.slot[i], src, bytes);
    if ((e = cudaMemcpyAsync(dst, g.slot[i], bytes, cudaMemcpyHostToDevice, st)) != cudaSuccess) return e;
    g.used[i] = true;
    return cudaEventRecord(g.done[i], st);
}

// Every upload goes through the staging slots, in slot-sized pieces, so the host source may be
// released as soon as this returns (nothing reads it later).
cudaError_t upload(void* dst, const void* src, size_t bytes, cudaStream_t st) {
    int dev = -1;
    Staging* gp = cudaGetDevice(&dev) == cudaSuccess ? staging(dev) : nullptr;
    if (!gp) return cudaMemcpyAsync(dst, src, bytes, cudaMemcpyHostToDevice, st);
    for (size_t off = 0; off < bytes; off += kStageSlotBytes) {
        const size_t n = std::min(kStageSlotBytes, bytes - off);
        cudaError_t e = upload_slot(*gp, static_cast<char*>(dst) + off, static_cast<const char*>(src) + off, n, st);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}
constexpr int kUnitKeys = 2048;            // automatic split: keys per unit (per KV head), at most
constexpr int64_t kMlaUnitCost = 256;      // an MLA unit's fixed start and end, in keys of streaming

struct SchedKey {
    int mla, dtype, hq, hkv, d, dv, pr, causal, window, path, kv_chunk;
    int sparse_bs, sparse_w;  // sparse top-K: block size and selection width (0 = dense)
    bool operator==(const SchedKey& o) const { return std::memcmp(this, &o, sizeof o) == 0; }
};

struct Schedule {
    SchedKey key;
    std::vector<char> host;  // uploaded blob, kept alive for the asynchronous copy
    void* dev = nullptr;
    const pa::KvUnit* tc_units = nullptr;     // tensor-core decode kernel
    const pa::KvUnit* simt_units = nullptr;   // CUDA-core kernel
    const pa::CombineUnit* cunits = nullptr;
    const pa::PrefillUnit* punits = nullptr;  // tensor-core prefill kernel
    const pa::KvUnit* mla_units = nullptr;    // tensor-core MLA decode kernel (two CTAs per unit)
    int32_t n_tc = 0, n_simt = 0, n_comb = 0, n_pre = 0, n_mla = 0;
    int32_t tc_rows_max = 0;
    int64_t slots = 0;  // workspace parts
    int32_t kv_chunk = 0;
};

}  // namespace

struct pa_plan {
    int device = -1;
    int num_sms = 148;
    int32_t S = 0, Nq = 0, table_width = 0, page_size = 0, num_pages = 0;
    std::vector<pa::SeqInfo> seqs;
    std::vector<int32_t> bt;
    void* d_meta = nullptr;
    std::vector<char> meta_host;
    pa::SeqInfo* d_seqs = nullptr;
    int32_t* d_bt = nullptr;
    int* d_err = nullptr;  // kernels' error word (bounded waits that ran out)
    int32_t* d_q2seq = nullptr;  // sequence of each packed query row
    int writes_checked = 0;      // 0 unknown, 1 every query row owns a distinct cache slot, -1 not
    std::vector<std::unique_ptr<Schedule>> scheds;  // most recent last
    float* ws = nullptr;
    size_t ws_bytes = 0;
    int32_t* sel_ws = nullptr;  // checked, compacted sparse selection
    size_t sel_ws_bytes = 0;
    float* score_ws = nullptr;  // proxy block scores when the caller keeps none
    size_t score_ws_bytes = 0;
    // tensor-core backward: work lists for one group size (key tiles, then row blocks) and Drow
    void* bwd_dev = nullptr;
    int32_t bwd_group = 0, bwd_causal = -1, bwd_window = -1, bwd_nkey = 0, bwd_nrow = 0;
    size_t bwd_row_off = 0;
    int32_t bwd_nord = 0, bwd_nsums = 0;  // ordered key tiles; cache rows of the ordered pass
    size_t bwd_sums_off = 0, bwd_refs_off = 0;
    std::vector<std::vector<char>> bwd_host;  // host blobs of the uploads (kept with the plan)
    float* bwd_drow = nullptr;
    size_t bwd_drow_bytes = 0;
    float* bwd_scratch = nullptr;  // finished dK then dV rows of ordered key tiles
    size_t bwd_scratch_bytes = 0;
    int* merge_ctr = nullptr;  // arrival counters of the decode kernel's own merge, zero between calls
    size_t merge_ctr_n = 0;
    // tensor-core MLA backward: key tiles and dQ units for one (heads, causal, window), the dS' scratch
    void* mla_bwd_dev = nullptr;
    int32_t mla_bwd_h = 0, mla_bwd_causal = -1, mla_bwd_window = -1, mla_ntiles = 0, mla_ndq = 0;
    size_t mla_dq_off = 0;
    int64_t mla_ds_cols = 0;
    std::vector<char> mla_bwd_host;
    void* mla_ds = nullptr;
    size_t mla_ds_bytes = 0;
    int shared_pages = -1;  // -1 unknown, 0 every used page belongs to one sequence once, 1 some page is shared
    cudaStream_t last_stream = nullptr;  // stream of the last call: frees are ordered on it
    int32_t last_launches = 0;
    int32_t last_kernels = 0;  // PA_KERNEL_* bits of the last call
    int64_t uploaded_bytes = 0;
    std::mutex mu;
};

namespace {

// ---------------------------------------------------------------------------------------
// Schedule construction
// ---------------------------------------------------------------------------------------

// Keys [lo, hi) that queries j0 .. j1-1 of a sequence can see (union over those queries).
void visible_union(int32_t L, int32_t n, int32_t j0, int32_t j1, bool causal, int32_t window,
                   int32_t* lo, int32_t* hi) {
    const int64_t p_first = (int64_t)L - n + j0;
    const int64_t p_last = (int64_t)L - n + j1 - 1;
    int64_t a = window > 0 ? std::max<int64_t>(0, p_first - window + 1) : 0;
    int64_t b = causal ? std::min<int64_t>(L, p_last + 1) : L;
    if (b < a) b = a;
    *lo = (int32_t)a;
    *hi = (int32_t)b;
}

int32_t ceil_div(int64_t a, int64_t b) { return (int32_t)((a + b - 1) / b); }

// Part length for the tensor-core MLA kernel. It runs one CTA per SM and two CTAs per unit, and
// the block scheduler hands the units (sorted longest first) to SM pairs as they free up. A unit
// costs about its keys plus kMlaUnitCost (loading the query rows, writing and merging its part),
// so among the lengths that fill one to eight waves of pairs this takes the one whose greedy
// longest-first hand-out is estimated to finish first (the shortest on a tie). Lengths are
// multiples of 64 keys, at least 256, and cut a range into at most kMaxSplits parts, like the
// units the schedule then builds.
int64_t mla_part_length(const std::vector<int64_t>& lens, int64_t total, int pairs) {
    pairs = std::max(1, pairs);
    int64_t best = 0, best_end = INT64_MAX;
    std::vector<int64_t> units, busy;
    for (int waves = 1; waves <= 8; ++waves) {
        int64_t c = (total + (int64_t)waves * pairs - 1) / ((int64_t)waves * pairs);
        c = std::max<int64_t>((c + 63) / 64 * 64, 256);
        units.clear();
        for (int64_t len : lens) {
            int64_t cc = c;
            if (len > cc * kMaxSplits) cc = (len + kMaxSplits - 1) / kMaxSplits;
            if (len <= 0) { units.push_back(0); continue; }
            for (int64_t t = 0; t < len; t += cc) units.push_back(std::min(cc, len - t));
        }
        std::sort(units.begin(), units.end(), std::greater<int64_t>());
        busy.assign(pairs, 0);  // min-heap of the times at which each pair frees up
        int64_t end = 0;
        for (int64_t u : units) {
            std::pop_heap(busy.begin(), busy.end(), std::greater<int64_t>());
            busy.back() += u + kMlaUnitCost;
            end = std::max(end, busy.back());
            std::push_heap(busy.begin(), busy.end(), std::greater<int64_t>());
        }
        if (end < best_end || (end == best_end && c < best)) { best_end = end; best = c; }
    }
    return best;
}

pa_status build_schedule(pa_plan* P, const SchedKey& k, cudaStream_t st, Schedule** out) {
    for (auto& s : P->scheds)
        if (s->key == k) { *out = s.get(); return PA_OK; }

    auto S = std::make_unique<Schedule>();
    S->key = k;
    const int32_t G = k.hq / k.hkv;
    const bool tc_decode = !k.mla && k.path == PA_PATH_AUTO && k.dtype != PA_F32 &&
                           k.d == k.dv && (k.d == 64 || k.d == 128 || k.d == 256);
    const bool tc_prefill = !k.mla && k.path == PA_PATH_AUTO &&
                            pa::prefill_tc_supported((pa_dtype)k.dtype, k.d, k.dv, G, P->page_size);
    const bool tc_mla = k.mla && k.path == PA_PATH_AUTO &&
                        pa::mla_tc_supported((pa_dtype)k.dtype, k.hq, k.d, k.pr, P->page_size);
    std::vector<pa::PrefillUnit> pu;
    std::vector<int64_t> pu_cost;

    struct Block { int32_t seq, j0, j1, lo, hi; int kind; };  // kind: 0 CUDA-core, 1 decode, 2 MLA
    std::vector<Block> blocks;
    int64_t total = 0;  // keys x kv heads, over all blocks
    // Sparse top-K: every query is its own row set; its keys are the concatenation of up to
    // sparse_w selected blocks (positions through the selection, see AttnParams::sel).
    const bool tc_sparse = tc_decode && G <= pa::kDecodeMaxRows && k.sparse_bs % 16 == 0;
    for (int32_t s = 0; k.sparse_bs > 0 && s < P->S; ++s) {
        const pa::SeqInfo& si = P->seqs[s];
        const int64_t nb = ((int64_t)si.L + k.sparse_bs - 1) / k.sparse_bs;
        const int64_t w = std::min<int64_t>(k.sparse_w, nb);
        for (int32_t j = 0; j < si.n; ++j) {
            Block b{s, j, j + 1, 0, (int32_t)(w * k.sparse_bs), tc_sparse ? 1 : 0};
            total += (int64_t)b.hi * k.hkv;
            blocks.push_back(b);
        }
    }
    for (int32_t s = 0; k.sparse_bs == 0 && s < P->S; ++s) {
        const pa::SeqInfo& si = P->seqs[s];
        if (si.n == 0) continue;
        const bool tc = tc_decode && (int64_t)si.n * G <= pa::kDecodeMaxRows;
        const bool mla_one = tc_mla && si.n == 1;
        if (!tc && !mla_one && tc_prefill) {
            // 128-row tiles: 128 / G queries times the G heads of one KV head
            const int32_t qpt = 128 / G;
            for (int32_t j0 = 0; j0 < si.n; j0 += qpt) {
                int32_t lo, hi;
                visible_union(si.L, si.n, j0, std::min(si.n, j0 + qpt), k.causal, k.window, &lo, &hi);
                for (int32_t h = 0; h < k.hkv; ++h) {
                    pa::PrefillUnit u{};
                    u.seq = s;
                    u.j0 = j0;
                    u.t0 = lo;
                    u.t1 = hi;
                    u.kvh = h;
                    pu.push_back(u);
                    pu_cost.push_back((int64_t)(hi - lo) + 128);
                }
            }
            continue;
        }
        // CUDA-core blocks take few queries so that long prefill chunks spread over CTAs.
        const int32_t qb = (tc || mla_one) ? si.n : std::max<int32_t>(1, 16 / std::min<int32_t>(G, 16));
        for (int32_t j0 = 0; j0 < si.n; j0 += qb) {
            Block b{s, j0, std::min(si.n, j0 + qb), 0, 0, tc ? 1 : (mla_one ? 2 : 0)};
            visible_union(si.L, si.n, b.j0, b.j1, k.causal, k.window, &b.lo, &b.hi);
            total += (int64_t)(b.hi - b.lo) * (k.mla ? 1 : k.hkv);
            blocks.push_back(b);
        }
    }
    int64_t chunk;
    if (k.kv_chunk > 0) chunk = k.sparse_bs > 0 ? ((int64_t)k.kv_chunk + 15) / 16 * 16 : k.kv_chunk;
    else if (k.kv_chunk < 0) chunk = INT32_MAX;
    else if (tc_mla) {
        std::vector<int64_t> lens;
        lens.reserve(blocks.size());
        for (const Block& b : blocks) lens.push_back(b.hi - b.lo);
        chunk = mla_part_length(lens, total, P->num_sms / 2);
    } else {
        // Long units amortise each CTA's start (first loads in flight) and end (merging its warps,
        // writing its part, merging the row): units of at most kUnitKeys keys (twice that for head
        // dims above 128, whose CTAs hold fewer tiles in flight), short enough that there are about
        // 7 units per 4 SMs, and never below 256 keys. Sparse rows are short runs of selected
        // blocks: whole rows up to 1024 keys per unit (no merge) beat finer splits.
        const int64_t unit_keys = (k.d > 128 || k.dv > 128) ? 2 * kUnitKeys : kUnitKeys;
        chunk = std::min<int64_t>(unit_keys, total * 4 / std::max<int64_t>(1, 7 * (int64_t)P->num_sms));
        chunk = std::max<int64_t>(((chunk + 63) / 64) * 64, k.sparse_bs > 0 ? 1024 : 256);
    }

    std::vector<pa::KvUnit> tcu, simtu, mlau;
    std::vector<pa::CombineUnit> cu;
    int64_t slots = 0;
    for (const Block& b : blocks) {
        const int64_t len = b.hi - b.lo;
        int64_t c = chunk;
        int32_t nsplit = len <= 0 ? 1 : ceil_div(len, c);
        if (nsplit > kMaxSplits) {
            c = (len + kMaxSplits - 1) / kMaxSplits;
            if (k.sparse_bs > 0) c = (c + 15) / 16 * 16;  // tiles of 16 keys stay inside one block
            nsplit = ceil_div(len, c);
        } else if (nsplit > 1 && k.kv_chunk == 0 && !tc_mla) {
            // automatic split: parts of (nearly) equal length, multiples of 64 keys, rather than
            // full parts and a short last one
            c = (ceil_div(len, nsplit) + 63) / 64 * 64;
            nsplit = ceil_div(len, c);
        }
        const int32_t base = nsplit > 1 ? (int32_t)slots : -1;
        if (nsplit > 1) {
            // the tensor-core decode kernel merges its own split rows (dense keys only); the merge
            // kernel takes the other kernels' rows
            if (!(b.kind == 1 && k.sparse_bs == 0))
                for (int32_t j = b.j0; j < b.j1; ++j)
                    cu.push_back({P->seqs[b.seq].q_start + j, base + (j - b.j0) * nsplit, nsplit, 0});
            slots += (int64_t)(b.j1 - b.j0) * nsplit;
        }
        for (int32_t i = 0; i < nsplit; ++i) {
            pa::KvUnit u;
            u.seq = b.seq;
            u.t0 = (int32_t)std::min<int64_t>(b.hi, b.lo + i * c);
            u.t1 = (int32_t)std::min<int64_t>(b.hi, b.lo + (i + 1) * c);
            u.split = i;
            u.nsplit = nsplit;
            u.part_base = base;
            u.j0 = b.j0;
            u.j1 = b.j1;
            (b.kind == 1 ? tcu : b.kind == 2 ? mlau : simtu).push_back(u);
            if (b.kind == 1) S->tc_rows_max = std::max<int32_t>(S->tc_rows_max, (b.j1 - b.j0) * G);
        }
    }
    // Longest units first: the block scheduler hands them out in index order.
    auto longer = [](const pa::KvUnit& a, const pa::KvUnit& b) {
        return (int64_t)(a.t1 - a.t0) * (a.j1 - a.j0) > (int64_t)(b.t1 - b.t0) * (b.j1 - b.j0);
    };
    std::stable_sort(tcu.begin(), tcu.end(), longer);
    std::stable_sort(simtu.begin(), simtu.end(), longer);
    std::stable_sort(mlau.begin(), mlau.end(), longer);
    {
        std::vector<size_t> order(pu.size());
        for (size_t i = 0; i < order.size(); ++i) order[i] = i;
        std::stable_sort(order.begin(), order.end(), [&](size_t a, size_t b) { return pu_cost[a] > pu_cost[b]; });
        std::vector<pa::PrefillUnit> sorted;
        sorted.reserve(pu.size());
        for (size_t i : order) sorted.push_back(pu[i]);
        pu.swap(sorted);
    }
    if (slots > INT32_MAX) return fail(PA_ERR_BOUNDS, "split workspace needs too many parts");

    // One blob: [tc units][simt units][combine units], 256-byte aligned sections.
    auto align = [](size_t x) { return (x + 255) & ~size_t(255); };
    const size_t o_tc = 0;
    const size_t o_simt = align(o_tc + tcu.size() * sizeof(pa::KvUnit));
    const size_t o_c = align(o_simt + simtu.size() * sizeof(pa::KvUnit));
    const size_t o_p = align(o_c + cu.size() * sizeof(pa::CombineUnit));
    const size_t o_m = align(o_p + pu.size() * sizeof(pa::PrefillUnit));
    const size_t bytes = align(o_m + mlau.size() * sizeof(pa::KvUnit));
    S->host.assign(std::max<size_t>(bytes, 256), 0);
    if (!tcu.empty()) std::memcpy(S->host.data() + o_tc, tcu.data(), tcu.size() * sizeof(pa::KvUnit));
    if (!simtu.empty()) std::memcpy(S->host.data() + o_simt, simtu.data(), simtu.size() * sizeof(pa::KvUnit));
    if (!cu.empty()) std::memcpy(S->host.data() + o_c, cu.data(), cu.size() * sizeof(pa::CombineUnit));
    if (!pu.empty()) std::memcpy(S->host.data() + o_p, pu.data(), pu.size() * sizeof(pa::PrefillUnit));
    if (!mlau.empty()) std::memcpy(S->host.data() + o_m, mlau.data(), mlau.size() * sizeof(pa::KvUnit));
    PA_CUDA_TRY(lib_malloc(&S->dev, S->host.size(), st));
    cudaError_t e = upload(S->dev, S->host.data(), S->host.size(), st);
    if (e != cudaSuccess) {
        lib_free(S->dev, P->device, st);
        return fail(PA_ERR_CUDA, "schedule upload failed: %s", cudaGetErrorString(e));
    }
    P->uploaded_bytes += (int64_t)S->host.size();
    char* base = (char*)S->dev;
    S->tc_units = (const pa::KvUnit*)(base + o_tc);
    S->simt_units = (const pa::KvUnit*)(base + o_simt);
    S->cunits = (const pa::CombineUnit*)(base + o_c);
    S->punits = (const pa::PrefillUnit*)(base + o_p);
    S->n_pre = (int32_t)pu.size();
    S->mla_units = (const pa::KvUnit*)(base + o_m);
    S->n_mla = (int32_t)mlau.size();
    S->n_tc = (int32_t)tcu.size();
    S->n_simt = (int32_t)simtu.size();
    S->n_comb = (int32_t)cu.size();
    S->slots = slots;
    S->kv_chunk = (int32_t)std::min<int64_t>(chunk, INT32_MAX);

    if (P->scheds.size() >= 8) {  // keep the plan's footprint bounded (stream-ordered free)
        lib_free(P->scheds.front()->dev, P->device, st);
        P->scheds.erase(P->scheds.begin());
    }
    P->scheds.push_back(std::move(S));
    *out = P->scheds.back().get();
    return PA_OK;
}

pa_status ensure_workspace(pa_plan* P, size_t bytes, cudaStream_t st) {
    if (bytes <= P->ws_bytes) return PA_OK;
    if (P->ws) {
        PA_CUDA_TRY(lib_free(P->ws, P->device, st));
        P->ws = nullptr;
        P->ws_bytes = 0;
    }
    void* p = nullptr;
    PA_CUDA_TRY(lib_malloc(&p, bytes, st));
    P->ws = (float*)p;
    P->ws_bytes = bytes;
    return PA_OK;
}

template <typename P_>
pa_status grow_buffer(P_** buf, size_t* have, size_t bytes, cudaStream_t st) {
    if (bytes <= *have) return PA_OK;
    if (*buf) {
        int dev = -1;
        PA_CUDA_TRY(cudaGetDevice(&dev));
        PA_CUDA_TRY(lib_free(*buf, dev, st));
        *buf = nullptr;
        *have = 0;
    }
    void* p = nullptr;
    PA_CUDA_TRY(lib_malloc(&p, bytes, st));
    *buf = (P_*)p;
    *have = bytes;
    return PA_OK;
}

// ---------------------------------------------------------------------------------------
// Shared validation of a forward call
// ---------------------------------------------------------------------------------------

struct Call {
    bool mla;
    const void *q, *k, *v, *qr, *kr;
    pa_dtype dtype;
    int32_t hq, hkv, d, dv, pr;
    float scale;
    int causal;
    int32_t window;
    void* out;
    float* lse;
    pa_forward_options opts;
    int32_t block_size;         // sparse top-K (0 = dense)
    const int32_t* selection;   // [Nq, Hkv, width]
    int32_t width;
};

int32_t max_blocks(const pa_plan* P, int32_t bs) {
    int64_t m = 0;
    for (const pa::SeqInfo& si : P->seqs) m = std::max<int64_t>(m, ((int64_t)si.L + bs - 1) / bs);
    return (int32_t)std::min<int64_t>(m, INT32_MAX);
}

// Block size rule and block count limit of the sparse entry points.
pa_status check_sparse_blocks(const pa_plan* P, int32_t bs) {
    if (bs <= 0 || bs % P->page_size != 0)
        return fail(PA_ERR_SHAPE, "block_size (%d) must be a positive multiple of page_size (%d)", bs, P->page_size);
    if (max_blocks(P, bs) > PA_SPARSE_MAX_BLOCKS)
        return fail(PA_ERR_UNSUPPORTED, "a sequence has more than %d blocks of %d keys", PA_SPARSE_MAX_BLOCKS, bs);
    return PA_OK;
}

pa_status validate(pa_plan* P, const Call& c) {
    if (!P) return fail(PA_ERR_INVALID_ARGUMENT, "plan is NULL");
    if (c.dtype != PA_F32 && c.dtype != PA_BF16 && c.dtype != PA_F16)
        return fail(PA_ERR_DTYPE, "unknown dtype %d", (int)c.dtype);
    if (c.hq <= 0 || c.hkv <= 0 || c.hq % c.hkv != 0)
        return fail(PA_ERR_SHAPE, "query heads (%d) must be a positive multiple of kv heads (%d)", c.hq, c.hkv);
    if (c.d <= 0 || c.dv <= 0)
        return fail(PA_ERR_SHAPE, "head dims must be positive (d=%d, dv=%d)", c.d, c.dv);
    if (c.d > 1024 || c.dv > 1024)
        return fail(PA_ERR_UNSUPPORTED, "head dims above 1024 are not supported (d=%d, dv=%d)", c.d, c.dv);
    if (c.mla && (c.pr <= 0 || c.pr > 256))
        return fail(PA_ERR_SHAPE, "MLA rope dim must be in 1..256 (got %d)", c.pr);
    if (!std::isfinite(c.scale) || !(c.scale > 0.0f))
        return fail(PA_ERR_INVALID_ARGUMENT, "scale must be finite and > 0");
    if (c.causal != 0 && c.causal != 1) return fail(PA_ERR_INVALID_ARGUMENT, "causal must be 0 or 1");
    if (c.window < 0) return fail(PA_ERR_INVALID_ARGUMENT, "window must be >= 0");
    if (c.opts.path != PA_PATH_AUTO && c.opts.path != PA_PATH_SIMT)
        return fail(PA_ERR_INVALID_ARGUMENT, "unknown path %d", c.opts.path);
    if (c.opts.kv_chunk < -1) return fail(PA_ERR_INVALID_ARGUMENT, "kv_chunk must be -1, 0 or > 0");
    if (c.block_size != 0) {
        pa_status bs = check_sparse_blocks(P, c.block_size);
        if (bs != PA_OK) return bs;
        if (c.width < 0) return fail(PA_ERR_SHAPE, "selection width must be >= 0");
    }

    const int64_t es = (int64_t)dtype_size(c.dtype);
    int64_t nq = P->Nq, pages = P->num_pages, ps = P->page_size;
    int64_t n_q, n_k, n_v, n_o, n_l, n_qr = 0, n_kr = 0;
    if (!product({nq, c.hq, c.d, es}, &n_q) || !product({pages, ps, c.hkv, c.d, es}, &n_k) ||
        !product({pages, ps, c.hkv, c.dv, es}, &n_v) || !product({nq, c.hq, c.dv, es}, &n_o) ||
        !product({nq, c.hq, 4}, &n_l) ||
        (c.mla && (!product({nq, c.hq, c.pr, es}, &n_qr) || !product({pages, ps, c.pr, es}, &n_kr))))
        return fail(PA_ERR_BOUNDS, "tensor size overflows 64-bit byte counts");
    if (nq == 0) return PA_OK;  // nothing is read or written
    if (!c.q || !c.out || !c.lse || (n_k > 0 && (!c.k || !c.v)) || (c.mla && (!c.qr || (n_kr > 0 && !c.kr))))
        return fail(PA_ERR_INVALID_ARGUMENT, "a required pointer is NULL");
    for (const void* ptr : {c.q, c.k, c.v, c.qr, c.kr, (const void*)c.out, (const void*)c.lse})
        if ((uintptr_t)ptr % 16 != 0)
            return fail(PA_ERR_INVALID_ARGUMENT, "device pointers must be 16-byte aligned");
    auto R = [](const void* p, int64_t n) { return Range{(uintptr_t)p, (uintptr_t)p + (uintptr_t)n}; };
    Range ro = R(c.out, n_o), rl = R(c.lse, n_l);
    Range ins[5] = {R(c.q, n_q), R(c.k, n_k), R(c.v, n_v), R(c.qr, n_qr), R(c.kr, n_kr)};
    if (overlap(ro, rl)) return fail(PA_ERR_ALIAS, "out and lse overlap");
    for (const Range& r : ins)
        if (overlap(ro, r) || overlap(rl, r)) return fail(PA_ERR_ALIAS, "out or lse overlaps an input");
    if (c.block_size > 0) {
        int64_t n_sel = 0;
        if (!product({nq, c.hkv, c.width, 4}, &n_sel)) return fail(PA_ERR_BOUNDS, "selection size overflows");
        if (n_sel > 0 && !c.selection) return fail(PA_ERR_INVALID_ARGUMENT, "selection is NULL");
        if ((uintptr_t)c.selection % 4 != 0) return fail(PA_ERR_INVALID_ARGUMENT, "selection must be 4-byte aligned");
        const Range rs = R(c.selection, n_sel);
        if (overlap(ro, rs) || overlap(rl, rs)) return fail(PA_ERR_ALIAS, "out or lse overlaps the selection");
    }
    return PA_OK;
}

pa_status run_forward(pa_plan* P, const Call& c, cudaStream_t st) {
    pa_status vs = validate(P, c);
    if (vs != PA_OK) return vs;
    if (P->Nq == 0) return ok();
    if (P->device < 0) return fail(PA_ERR_INVALID_ARGUMENT, "host-only plan: no device to run on");
    int cur = -1;
    PA_CUDA_TRY(cudaGetDevice(&cur));
    if (cur != P->device)
        return fail(PA_ERR_INVALID_ARGUMENT, "current device %d is not the plan's device %d", cur, P->device);

    std::lock_guard<std::mutex> lock(P->mu);
    P->last_stream = st;
    SchedKey key{};
    key.mla = c.mla;
    key.dtype = c.dtype;
    key.hq = c.hq;
    key.hkv = c.hkv;
    key.d = c.d;
    key.dv = c.dv;
    key.pr = c.mla ? c.pr : 0;
    key.causal = c.causal;
    key.window = c.window;
    key.path = c.opts.path;
    key.kv_chunk = c.opts.kv_chunk;
    int32_t wout = 0;  // width of the compacted selection
    if (c.block_size > 0) {
        wout = std::min<int32_t>(c.width, max_blocks(P, c.block_size));
        key.sparse_bs = c.block_size;
        key.sparse_w = wout;
    }
    Schedule* S = nullptr;
    pa_status bs = build_schedule(P, key, st, &S);
    if (bs != PA_OK) return bs;
    if (c.block_size > 0 && wout > 0) {
        pa_status gs = grow_buffer(&P->sel_ws, &P->sel_ws_bytes, (size_t)P->Nq * c.hkv * wout * sizeof(int32_t), st);
        if (gs != PA_OK) return gs;
    }
    if (S->slots > 0) {
        const size_t need = (size_t)S->slots * c.hq * (c.dv + 1) * sizeof(float);
        pa_status ws = ensure_workspace(P, need, st);
        if (ws != PA_OK) return ws;
    }

    pa::AttnParams p{};
    p.q = c.q; p.k = c.k; p.v = c.v; p.qr = c.qr; p.kr = c.kr;
    p.out = c.out; p.lse = c.lse;
    p.ws_o = P->ws;
    p.ws_lse = P->ws ? P->ws + (size_t)S->slots * c.hq * c.dv : nullptr;
    p.seqs = P->d_seqs;
    p.block_tables = P->d_bt;
    p.cunits = S->cunits;
    p.num_cunits = S->n_comb;
    p.table_width = P->table_width;
    p.page_size = P->page_size;
    p.hq = c.hq; p.hkv = c.hkv; p.group = c.hq / c.hkv;
    p.d = c.d; p.dv = c.dv; p.pr = c.mla ? c.pr : 0;
    p.scale = c.scale;
    p.scale_log2 = (float)((double)c.scale * 1.4426950408889634);
    p.causal = c.causal; p.window = c.window;
    p.num_queries = P->Nq;
    p.num_pages = P->num_pages;
    p.err = P->d_err;
    p.punits = S->punits;
    p.num_punits = S->n_pre;

    cudaEvent_t* ev = (cudaEvent_t*)c.opts.trace_events;
    cudaError_t e;
    int launches = 0;
    uint32_t kernels = 0;
    if (c.block_size > 0) {
        p.sel = P->sel_ws;
        p.sel_width = wout;
        p.block_size = c.block_size;
        if (wout > 0) {
            ++launches;
            kernels |= PA_KERNEL_SPARSE;
            e = pa::launch_sparse_prep(c.selection, c.width, P->sel_ws, wout, P->d_seqs, P->d_q2seq, c.hkv,
                                       c.block_size, max_blocks(P, c.block_size), P->Nq, P->d_err, st);
            if (e != cudaSuccess) return fail(PA_ERR_CUDA, "selection check launch failed: %s", cudaGetErrorString(e));
        }
    }
    if (S->n_tc > 0 && S->slots > 0 && c.block_size == 0) {
        // counters of the decode kernel's own merge: zeroed when allocated, and put back to zero by
        // the kernel after each merge, so every call finds them zero
        const size_t n = (size_t)S->slots * c.hkv;
        if (n > P->merge_ctr_n) {
            if (P->merge_ctr) PA_CUDA_TRY(lib_free(P->merge_ctr, P->device, st));
            P->merge_ctr = nullptr;
            P->merge_ctr_n = 0;
            void* m = nullptr;
            PA_CUDA_TRY(lib_malloc(&m, n * sizeof(int), st));
            PA_CUDA_TRY(cudaMemsetAsync(m, 0, n * sizeof(int), st));
            P->merge_ctr = (int*)m;
            P->merge_ctr_n = n;
        }
        p.merge_ctr = P->merge_ctr;
    }
    if (ev) PA_CUDA_TRY(cudaEventRecord(ev[0], st));
    {
        // Decode rows beside prefill chunks: the persistent prefill kernel on the caller's stream,
        // then the decode kernel on the library's side stream (forked and joined through events),
        // so that decode CTAs take the SMs the prefill CTAs leave as they finish (C4: 3-4 % faster
        // than the two in series).
        const bool fork = S->n_tc > 0 && S->n_pre > 0;
        std::unique_lock<std::mutex> side_lock(pa::side_mutex(), std::defer_lock);
        pa::SideStream* side = nullptr;
        if (fork) {
            side_lock.lock();
            e = pa::side_stream(&side);
            if (e == cudaSuccess) e = cudaEventRecord(side->fork, st);
            if (e == cudaSuccess) e = cudaStreamWaitEvent(side->stream, side->fork, 0);
            if (e != cudaSuccess) return fail(PA_ERR_CUDA, "side stream fork failed: %s", cudaGetErrorString(e));
        }
        const char* what = nullptr;
        if (S->n_pre > 0) {
            ++launches;
            kernels |= PA_KERNEL_PREFILL_TC;
            e = pa::launch_prefill_tc(p, c.dtype, P->num_pages, st);
            if (e != cudaSuccess) what = "prefill kernel launch";
        }
        if (!what && S->n_tc > 0) {
            ++launches;
            kernels |= PA_KERNEL_DECODE_TC;
            p.units = S->tc_units;
            p.num_units = S->n_tc;
            e = pa::launch_decode_mma(p, c.dtype, S->tc_rows_max, fork ? side->stream : st);
            if (e != cudaSuccess) what = "decode kernel launch";
        }
        if (fork) {  // joined on every path, so that a capture on the caller's stream never ends unjoined
            cudaError_t j = cudaEventRecord(side->join, side->stream);
            if (j == cudaSuccess) j = cudaStreamWaitEvent(st, side->join, 0);
            if (!what && j != cudaSuccess) {
                e = j;
                what = "side stream join";
            }
        }
        if (what) return fail(PA_ERR_CUDA, "%s failed: %s", what, cudaGetErrorString(e));
    }
    if (S->n_mla > 0) {
        ++launches;
        kernels |= PA_KERNEL_MLA_TC;
        p.units = S->mla_units;
        p.num_units = S->n_mla;
        e = pa::launch_mla_tc(p, c.dtype, st);
        if (e != cudaSuccess) return fail(PA_ERR_CUDA, "MLA kernel launch failed: %s", cudaGetErrorString(e));
    }
    if (S->n_simt > 0) {
        ++launches;
        kernels |= PA_KERNEL_SIMT;
        p.units = S->simt_units;
        p.num_units = S->n_simt;
        e = pa::launch_simt(p, c.dtype, st);
        if (e != cudaSuccess) return fail(PA_ERR_CUDA, "CUDA-core kernel launch failed: %s", cudaGetErrorString(e));
    }
    if (ev) PA_CUDA_TRY(cudaEventRecord(ev[1], st));
    if (S->n_comb > 0) {
        ++launches;
        kernels |= PA_KERNEL_MERGE;
        e = pa::launch_combine(p, c.dtype, st);
        if (e != cudaSuccess) return fail(PA_ERR_CUDA, "combine kernel launch failed: %s", cudaGetErrorString(e));
    }
    if (ev) PA_CUDA_TRY(cudaEventRecord(ev[2], st));
    P->last_launches = launches;
    P->last_kernels = (int32_t)kernels;
    return ok();
}

pa_forward_options default_opts(const pa_forward_options* o) {
    pa_forward_options d{0, PA_PATH_AUTO, nullptr};
    return o ? *o : d;
}

}  // namespace

namespace pa {

pa_status set_error(pa_status st, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_msg, sizeof g_msg, fmt, ap);
    va_end(ap);
    return st;
}

pa_status clear_error() { return ok(); }

pa_status validated_gqa_view(pa_plan* P, const void* q, const void* k, const void* v, pa_dtype dtype, int32_t hq,
                             int32_t hkv, int32_t d, int32_t dv, float scale, int causal, int32_t window,
                             void* out, float* lse, PlanView* view) {
    Call c{};
    c.mla = false;
    c.q = q; c.k = k; c.v = v;
    c.dtype = dtype;
    c.hq = hq; c.hkv = hkv; c.d = d; c.dv = dv;
    c.scale = scale; c.causal = causal; c.window = window;
    c.out = out; c.lse = lse;
    c.opts = default_opts(nullptr);
    pa_status vs = validate(P, c);
    if (vs != PA_OK) return vs;
    if (P->Nq > 0) {
        if (P->device < 0) return fail(PA_ERR_INVALID_ARGUMENT, "host-only plan: no device to run on");
        int cur = -1;
        PA_CUDA_TRY(cudaGetDevice(&cur));
        if (cur != P->device)
            return fail(PA_ERR_INVALID_ARGUMENT, "current device %d is not the plan's device %d", cur, P->device);
    }
    view->device = P->device;
    view->num_sms = P->num_sms;
    view->S = P->S;
    view->Nq = P->Nq;
    view->table_width = P->table_width;
    view->page_size = P->page_size;
    view->num_pages = P->num_pages;
    view->host_seqs = P->seqs.data();
    view->d_seqs = P->d_seqs;
    view->d_bt = P->d_bt;
    view->d_err = P->d_err;
    return PA_OK;
}

}  // namespace pa

// ---------------------------------------------------------------------------------------
// C ABI
// ---------------------------------------------------------------------------------------

extern "C" {

pa_status pa_plan_create(const int32_t* seq_lens, const int32_t* query_offsets, int32_t num_seqs,
                         const int32_t* block_tables, int32_t table_width, int32_t page_size,
                         int32_t num_pages, int device, pa_stream upload_stream, pa_plan** out_plan) {
    if (!out_plan) return fail(PA_ERR_INVALID_ARGUMENT, "out_plan is NULL");
    *out_plan = nullptr;
    if (num_seqs < 0) return fail(PA_ERR_INVALID_ARGUMENT, "num_seqs must be >= 0");
    if (page_size <= 0) return fail(PA_ERR_INVALID_ARGUMENT, "page_size must be > 0");
    if (num_pages < 0 || table_width < 0)
        return fail(PA_ERR_INVALID_ARGUMENT, "num_pages and table_width must be >= 0");
    if (device < -1) return fail(PA_ERR_INVALID_ARGUMENT, "device must be >= -1");
    if (!query_offsets) return fail(PA_ERR_INVALID_ARGUMENT, "query_offsets is NULL");
    if (num_seqs > 0 && !seq_lens) return fail(PA_ERR_INVALID_ARGUMENT, "seq_lens is NULL");
    if (query_offsets[0] != 0) return fail(PA_ERR_INVALID_ARGUMENT, "query_offsets[0] must be 0");
    int64_t bt_elems = 0;
    if (!product({num_seqs, table_width}, &bt_elems) || bt_elems > INT32_MAX)
        return fail(PA_ERR_BOUNDS, "block table too large");
    for (int32_t s = 0; s < num_seqs; ++s) {
        const int64_t L = seq_lens[s];
        const int64_t n = (int64_t)query_offsets[s + 1] - query_offsets[s];
        if (L < 0) return fail(PA_ERR_INVALID_ARGUMENT, "seq_lens[%d] = %lld < 0", s, (long long)L);
        if (n < 0) return fail(PA_ERR_INVALID_ARGUMENT, "query_offsets decrease at sequence %d", s);
        if (n > L) return fail(PA_ERR_INVALID_ARGUMENT, "sequence %d has %lld queries but only %lld keys", s, (long long)n, (long long)L);
        const int64_t used = (L + page_size - 1) / page_size;
        if (used > table_width)
            return fail(PA_ERR_BOUNDS, "sequence %d needs %lld pages but table_width is %d", s, (long long)used, table_width);
        if (used > 0 && !block_tables) return fail(PA_ERR_INVALID_ARGUMENT, "block_tables is NULL");
        for (int64_t b = 0; b < used; ++b) {
            const int32_t pg = block_tables[(int64_t)s * table_width + b];
            if (pg < 0 || pg >= num_pages)
                return fail(PA_ERR_BOUNDS, "block_tables[%d][%lld] = %d is outside the pool [0, %d)", s, (long long)b, pg, num_pages);
        }
    }
    const int64_t nq = query_offsets[num_seqs];
    if (nq > INT32_MAX) return fail(PA_ERR_BOUNDS, "too many queries");

    auto P = std::make_unique<pa_plan>();
    P->device = device;
    P->S = num_seqs;
    P->Nq = (int32_t)nq;
    P->table_width = table_width;
    P->page_size = page_size;
    P->num_pages = num_pages;
    P->seqs.resize(num_seqs);
    for (int32_t s = 0; s < num_seqs; ++s)
        P->seqs[s] = {seq_lens[s], query_offsets[s], query_offsets[s + 1] - query_offsets[s], 0};
    if (bt_elems > 0) {
        if (!block_tables) return fail(PA_ERR_INVALID_ARGUMENT, "block_tables is NULL");
        P->bt.assign(block_tables, block_tables + bt_elems);
    }

    if (device >= 0) {
        int cur = -1;
        PA_CUDA_TRY(cudaGetDevice(&cur));
        if (cur != device) return fail(PA_ERR_INVALID_ARGUMENT, "current device %d is not %d", cur, device);
        PA_CUDA_TRY(cudaDeviceGetAttribute(&P->num_sms, cudaDevAttrMultiProcessorCount, device));
        const size_t seq_bytes = ((sizeof(pa::SeqInfo) * num_seqs + 255) / 256) * 256;
        const size_t bt_bytes = ((sizeof(int32_t) * (size_t)bt_elems + 255) / 256) * 256;
        const size_t q2s_bytes = ((sizeof(int32_t) * (size_t)nq + 255) / 256) * 256;
        const size_t total = seq_bytes + bt_bytes + 256 + q2s_bytes;  // + the error word + query->sequence
        std::vector<char>& blob = P->meta_host;  // kept alive for the asynchronous copy
        blob.assign(total, 0);
        if (num_seqs) std::memcpy(blob.data(), P->seqs.data(), sizeof(pa::SeqInfo) * num_seqs);
        if (bt_elems) std::memcpy(blob.data() + seq_bytes, P->bt.data(), sizeof(int32_t) * (size_t)bt_elems);
        {
            int32_t* q2s = reinterpret_cast<int32_t*>(blob.data() + seq_bytes + bt_bytes + 256);
            for (int32_t s = 0; s < num_seqs; ++s)
                for (int32_t q = query_offsets[s]; q < query_offsets[s + 1]; ++q) q2s[q] = s;
        }
        PA_CUDA_TRY(lib_malloc(&P->d_meta, total, (cudaStream_t)upload_stream));
        cudaError_t e = upload(P->d_meta, blob.data(), total, (cudaStream_t)upload_stream);
        P->last_stream = (cudaStream_t)upload_stream;
        P->uploaded_bytes = (int64_t)total;
        if (e != cudaSuccess) {
            lib_free(P->d_meta, device, (cudaStream_t)upload_stream);
            return fail(PA_ERR_CUDA, "plan upload failed: %s", cudaGetErrorString(e));
        }
        P->d_seqs = (pa::SeqInfo*)P->d_meta;
        P->d_bt = (int32_t*)((char*)P->d_meta + seq_bytes);
        P->d_err = (int*)((char*)P->d_meta + seq_bytes + bt_bytes);
        P->d_q2seq = (int32_t*)((char*)P->d_meta + seq_bytes + bt_bytes + 256);
    }
    *out_plan = P.release();
    return ok();
}

pa_status pa_plan_destroy(pa_plan* plan) {
    if (!plan) return ok();
    if (plan->device >= 0) {
        // Stream-ordered frees after the plan's last queued use. Uploads read page-locked copies of
        // the plan's host data, never the plan's own buffers, so the plan object goes at once (no
        // host callback on the stream, which would hold back the work queued after it).
        cudaStream_t st = plan->last_stream;
        const int dv = plan->device;
        lib_free(plan->ws, dv, st);
        lib_free(plan->sel_ws, dv, st);
        lib_free(plan->score_ws, dv, st);
        lib_free(plan->bwd_dev, dv, st);
        lib_free(plan->bwd_drow, dv, st);
        lib_free(plan->bwd_scratch, dv, st);
        lib_free(plan->merge_ctr, dv, st);
        lib_free(plan->mla_bwd_dev, dv, st);
        lib_free(plan->mla_ds, dv, st);
        for (auto& s : plan->scheds) lib_free(s->dev, dv, st);
        cudaError_t e = lib_free(plan->d_meta, dv, st);
        delete plan;
        if (e != cudaSuccess) return fail(PA_ERR_CUDA, "plan release failed: %s", cudaGetErrorString(e));
        return ok();
    }
    delete plan;
    return ok();
}

pa_status pa_plan_get_info(const pa_plan* plan, pa_plan_info* info) {
    if (!plan || !info) return fail(PA_ERR_INVALID_ARGUMENT, "plan or info is NULL");
    info->num_seqs = plan->S;
    info->num_queries = plan->Nq;
    info->table_width = plan->table_width;
    info->page_size = plan->page_size;
    info->num_pages = plan->num_pages;
    info->device = plan->device;
    info->last_launches = plan->last_launches;
    info->workspace_bytes = (int64_t)plan->ws_bytes;
    info->uploaded_bytes = plan->uploaded_bytes;
    info->last_kernels = plan->last_kernels;
    return ok();
}

pa_status pa_forward_ex(pa_plan* plan, const void* q, const void* k_cache, const void* v_cache,
                        pa_dtype dtype, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                        int32_t v_head_dim, float scale, int causal, int32_t window, void* out,
                        float* lse, pa_stream stream, const pa_forward_options* opts) {
    Call c{};
    c.mla = false;
    c.q = q; c.k = k_cache; c.v = v_cache;
    c.dtype = dtype;
    c.hq = num_q_heads; c.hkv = num_kv_heads; c.d = head_dim; c.dv = v_head_dim;
    c.scale = scale; c.causal = causal; c.window = window;
    c.out = out; c.lse = lse;
    c.opts = default_opts(opts);
    return run_forward(plan, c, (cudaStream_t)stream);
}

pa_status pa_forward(pa_plan* plan, const void* q, const void* k_cache, const void* v_cache,
                     pa_dtype dtype, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                     int32_t v_head_dim, float scale, int causal, int32_t window, void* out,
                     float* lse, pa_stream stream) {
    return pa_forward_ex(plan, q, k_cache, v_cache, dtype, num_q_heads, num_kv_heads, head_dim,
                         v_head_dim, scale, causal, window, out, lse, stream, nullptr);
}

pa_status pa_mla_forward_ex(pa_plan* plan, const void* q_latent, const void* q_rope,
                            const void* latent_cache, const void* rope_cache, pa_dtype dtype,
                            int32_t num_heads, int32_t latent_dim, int32_t rope_dim, float scale,
                            int causal, int32_t window, void* out, float* lse, pa_stream stream,
                            const pa_forward_options* opts) {
    Call c{};
    c.mla = true;
    c.q = q_latent; c.k = latent_cache; c.v = latent_cache; c.qr = q_rope; c.kr = rope_cache;
    c.dtype = dtype;
    c.hq = num_heads; c.hkv = 1; c.d = latent_dim; c.dv = latent_dim; c.pr = rope_dim;
    c.scale = scale; c.causal = causal; c.window = window;
    c.out = out; c.lse = lse;
    c.opts = default_opts(opts);
    return run_forward(plan, c, (cudaStream_t)stream);
}

pa_status pa_mla_forward(pa_plan* plan, const void* q_latent, const void* q_rope,
                         const void* latent_cache, const void* rope_cache, pa_dtype dtype,
                         int32_t num_heads, int32_t latent_dim, int32_t rope_dim, float scale,
                         int causal, int32_t window, void* out, float* lse, pa_stream stream) {
    return pa_mla_forward_ex(plan, q_latent, q_rope, latent_cache, rope_cache, dtype, num_heads,
                             latent_dim, rope_dim, scale, causal, window, out, lse, stream, nullptr);
}

pa_status pa_sparse_forward(pa_plan* plan, const void* q, const void* k_cache, const void* v_cache,
                            pa_dtype dtype, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                            int32_t v_head_dim, float scale, int causal, int32_t window, int32_t block_size,
                            const int32_t* selection, int32_t width, void* out, float* lse, pa_stream stream) {
    return pa_sparse_forward_ex(plan, q, k_cache, v_cache, dtype, num_q_heads, num_kv_heads, head_dim, v_head_dim,
                                scale, causal, window, block_size, selection, width, out, lse, stream, nullptr);
}

pa_status pa_sparse_forward_ex(pa_plan* plan, const void* q, const void* k_cache, const void* v_cache,
                               pa_dtype dtype, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                               int32_t v_head_dim, float scale, int causal, int32_t window, int32_t block_size,
                               const int32_t* selection, int32_t width, void* out, float* lse, pa_stream stream,
                               const pa_forward_options* opts) {
    if (!plan) return fail(PA_ERR_INVALID_ARGUMENT, "plan is NULL");
    if (block_size <= 0) return fail(PA_ERR_SHAPE, "block_size must be > 0");
    Call c{};
    c.mla = false;
    c.q = q; c.k = k_cache; c.v = v_cache;
    c.dtype = dtype;
    c.hq = num_q_heads; c.hkv = num_kv_heads; c.d = head_dim; c.dv = v_head_dim;
    c.scale = scale; c.causal = causal; c.window = window;
    c.out = out; c.lse = lse;
    c.opts = default_opts(opts);
    c.block_size = block_size;
    c.selection = selection;
    c.width = width;
    return run_forward(plan, c, (cudaStream_t)stream);
}

pa_status pa_sparse_select(pa_plan* plan, const void* q, const void* k_cache, pa_dtype dtype,
                           int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim, float scale,
                           int causal, int32_t window, int32_t block_size, int32_t topk,
                           int32_t* selection, int32_t width, float* block_scores, int32_t scores_width,
                           pa_stream stream) {
    pa_plan* P = plan;
    if (!P) return fail(PA_ERR_INVALID_ARGUMENT, "plan is NULL");
    if (dtype != PA_F32 && dtype != PA_BF16 && dtype != PA_F16) return fail(PA_ERR_DTYPE, "unknown dtype %d", (int)dtype);
    if (num_q_heads <= 0 || num_kv_heads <= 0 || num_q_heads % num_kv_heads != 0)
        return fail(PA_ERR_SHAPE, "query heads (%d) must be a positive multiple of kv heads (%d)", num_q_heads,
                    num_kv_heads);
    if (head_dim <= 0) return fail(PA_ERR_SHAPE, "head_dim must be positive");
    if (head_dim > 1024) return fail(PA_ERR_UNSUPPORTED, "head dims above 1024 are not supported");
    if (!std::isfinite(scale) || !(scale > 0.0f)) return fail(PA_ERR_INVALID_ARGUMENT, "scale must be finite and > 0");
    if (causal != 0 && causal != 1) return fail(PA_ERR_INVALID_ARGUMENT, "causal must be 0 or 1");
    if (window < 0) return fail(PA_ERR_INVALID_ARGUMENT, "window must be >= 0");
    if (topk < 0) return fail(PA_ERR_INVALID_ARGUMENT, "topk must be >= 0");
    pa_status bst = check_sparse_blocks(P, block_size);
    if (bst != PA_OK) return bst;
    const int32_t nb_max = max_blocks(P, block_size);
    int64_t k_max = 0;
    for (const pa::SeqInfo& si : P->seqs) {
        if (si.n == 0) continue;
        const int64_t nb = ((int64_t)si.L + block_size - 1) / block_size;
        k_max = std::max<int64_t>(k_max, (topk == 0 || topk >= nb) ? nb : topk);
    }
    if (width < k_max) return fail(PA_ERR_SHAPE, "selection width %d is below the %lld blocks kept", width, (long long)k_max);
    if (block_scores && scores_width < nb_max)
        return fail(PA_ERR_SHAPE, "scores_width %d is below the %d blocks of the longest sequence", scores_width, nb_max);
    const int64_t es = (int64_t)dtype_size(dtype);
    int64_t n_q, n_k, n_sel, n_sc = 0;
    if (!product({P->Nq, num_q_heads, head_dim, es}, &n_q) ||
        !product({P->num_pages, P->page_size, num_kv_heads, head_dim, es}, &n_k) ||
        !product({P->Nq, num_kv_heads, width, 4}, &n_sel) ||
        (block_scores && !product({P->Nq, num_kv_heads, scores_width, 4}, &n_sc)))
        return fail(PA_ERR_BOUNDS, "tensor size overflows 64-bit byte counts");
    if (P->Nq == 0) return ok();
    if (!q || (n_k > 0 && !k_cache) || (n_sel > 0 && !selection))
        return fail(PA_ERR_INVALID_ARGUMENT, "a required pointer is NULL");
    if ((uintptr_t)q % 16 || (uintptr_t)k_cache % 16 || (uintptr_t)selection % 4 || (uintptr_t)block_scores % 4)
        return fail(PA_ERR_INVALID_ARGUMENT, "q and k_cache must be 16-byte aligned, selection and scores 4-byte");
    auto R = [](const void* p, int64_t n) { return Range{(uintptr_t)p, (uintptr_t)p + (uintptr_t)n}; };
    const Range rq = R(q, n_q), rk = R(k_cache, n_k), rs = R(selection, n_sel), rc = R(block_scores, n_sc);
    if (overlap(rs, rq) || overlap(rs, rk) || overlap(rc, rq) || overlap(rc, rk) || overlap(rs, rc))
        return fail(PA_ERR_ALIAS, "selection or block_scores overlaps an input or each other");
    if (P->device < 0) return fail(PA_ERR_INVALID_ARGUMENT, "host-only plan: no device to run on");
    int cur = -1;
    PA_CUDA_TRY(cudaGetDevice(&cur));
    if (cur != P->device) return fail(PA_ERR_INVALID_ARGUMENT, "current device %d is not the plan's device %d", cur, P->device);

    std::lock_guard<std::mutex> lock(P->mu);
    cudaStream_t st = (cudaStream_t)stream;
    P->last_stream = st;
    float* scores = block_scores;
    int32_t sw = scores_width;
    if (!scores) {
        sw = nb_max;
        pa_status gs = grow_buffer(&P->score_ws, &P->score_ws_bytes, std::max<size_t>(4, (size_t)P->Nq * num_kv_heads * sw * 4), st);
        if (gs != PA_OK) return gs;
        scores = P->score_ws;
    }
    cudaError_t e = pa::launch_sparse_scores(q, k_cache, scores, sw, P->d_seqs, P->d_q2seq, P->d_bt, P->table_width,
                                             P->page_size, num_q_heads, num_kv_heads, head_dim, block_size, scale,
                                             causal, window, P->Nq, dtype, st);
    if (e != cudaSuccess) return fail(PA_ERR_CUDA, "proxy score launch failed: %s", cudaGetErrorString(e));
    if (width > 0) {
        e = pa::launch_sparse_topk(scores, sw, selection, width, P->d_seqs, P->d_q2seq, num_kv_heads, block_size, topk,
                                   nb_max, P->Nq, st);
        if (e != cudaSuccess) return fail(PA_ERR_CUDA, "top-k launch failed: %s", cudaGetErrorString(e));
    }
    P->last_launches = width > 0 ? 2 : 1;
    P->last_kernels = PA_KERNEL_SPARSE;
    return ok();
}

pa_status pa_plan_prepare(pa_plan* plan, int mla, pa_dtype dtype, int32_t num_q_heads,
                          int32_t num_kv_heads, int32_t head_dim, int32_t v_head_dim, int causal,
                          int32_t window, pa_stream stream, const pa_forward_options* opts) {
    if (!plan) return fail(PA_ERR_INVALID_ARGUMENT, "plan is NULL");
    if (plan->device < 0) return fail(PA_ERR_INVALID_ARGUMENT, "host-only plan: no device to prepare");
    pa_forward_options o = default_opts(opts);
    SchedKey key{};
    key.mla = mla ? 1 : 0;
    key.dtype = dtype;
    key.hq = num_q_heads;
    key.hkv = mla ? 1 : num_kv_heads;
    key.d = head_dim;
    key.dv = mla ? head_dim : v_head_dim;
    key.pr = mla ? v_head_dim : 0;  // for MLA the fifth size argument is the rope width
    if (mla) key.dv = head_dim;
    key.causal = causal;
    key.window = window;
    key.path = o.path;
    key.kv_chunk = o.kv_chunk;
    if (key.hq <= 0 || key.hkv <= 0 || key.hq % key.hkv || key.d <= 0 || key.dv <= 0)
        return fail(PA_ERR_SHAPE, "inconsistent head configuration");
    std::lock_guard<std::mutex> lock(plan->mu);
    Schedule* S = nullptr;
    pa_status st = build_schedule(plan, key, (cudaStream_t)stream, &S);
    if (st != PA_OK) return st;
    if (S->slots > 0) {
        st = ensure_workspace(plan, (size_t)S->slots * key.hq * (key.dv + 1) * sizeof(float), (cudaStream_t)stream);
        if (st != PA_OK) return st;
    }
    return ok();
}

pa_status pa_append(pa_plan* plan, const void* new_k, const void* new_v, void* k_cache, void* v_cache,
                    pa_dtype dtype, int32_t num_kv_heads, int32_t head_dim, int32_t v_head_dim, pa_stream stream) {
    if (!plan) return fail(PA_ERR_INVALID_ARGUMENT, "plan is NULL");
    if (dtype != PA_F32 && dtype != PA_BF16 && dtype != PA_F16) return fail(PA_ERR_DTYPE, "unknown dtype %d", (int)dtype);
    if (num_kv_heads <= 0 || head_dim <= 0 || v_head_dim <= 0)
        return fail(PA_ERR_SHAPE, "kv heads and head dims must be positive");
    if (head_dim > 1024 || v_head_dim > 1024) return fail(PA_ERR_UNSUPPORTED, "head dims above 1024 are not supported");
    const int64_t es = (int64_t)dtype_size(dtype);
    const int64_t kb = head_dim * es, vb = v_head_dim * es;
    if (kb % 16 || vb % 16) return fail(PA_ERR_UNSUPPORTED, "rows must be multiples of 16 bytes (head_dim * element size)");
    int64_t n_new_k, n_new_v, n_k, n_v;
    if (!product({plan->Nq, num_kv_heads, kb}, &n_new_k) || !product({plan->Nq, num_kv_heads, vb}, &n_new_v) ||
        !product({plan->num_pages, plan->page_size, num_kv_heads, kb}, &n_k) ||
        !product({plan->num_pages, plan->page_size, num_kv_heads, vb}, &n_v))
        return fail(PA_ERR_BOUNDS, "tensor size overflows 64-bit byte counts");
    if (plan->Nq == 0) return ok();
    if (!new_k || !new_v || !k_cache || !v_cache) return fail(PA_ERR_INVALID_ARGUMENT, "a required pointer is NULL");
    for (const void* ptr : {new_k, new_v, (const void*)k_cache, (const void*)v_cache})
        if ((uintptr_t)ptr % 16 != 0) return fail(PA_ERR_INVALID_ARGUMENT, "device pointers must be 16-byte aligned");
    auto R = [](const void* p, int64_t n) { return Range{(uintptr_t)p, (uintptr_t)p + (uintptr_t)n}; };
    const Range rk = R(k_cache, n_k), rv = R(v_cache, n_v), rnk = R(new_k, n_new_k), rnv = R(new_v, n_new_v);
    if (overlap(rk, rv)) return fail(PA_ERR_ALIAS, "k_cache and v_cache overlap");
    if (overlap(rk, rnk) || overlap(rk, rnv) || overlap(rv, rnk) || overlap(rv, rnv))
        return fail(PA_ERR_ALIAS, "new rows overlap a cache");
    // Every query row must own a distinct cache slot, or two rows would race for one slot
    // (e.g. sequences sharing a prefix page). Checked once per plan.
    if (plan->writes_checked == 0) {
        std::vector<int64_t> slots;
        slots.reserve((size_t)plan->Nq);
        for (int32_t s = 0; s < plan->S; ++s) {
            const pa::SeqInfo& si = plan->seqs[s];
            for (int32_t j = 0; j < si.n; ++j) {
                const int64_t pos = (int64_t)si.L - si.n + j;
                slots.push_back((int64_t)plan->bt[(int64_t)s * plan->table_width + pos / plan->page_size] * plan->page_size +
                                pos % plan->page_size);
            }
        }
        std::sort(slots.begin(), slots.end());
        plan->writes_checked = std::adjacent_find(slots.begin(), slots.end()) == slots.end() ? 1 : -1;
    }
    if (plan->writes_checked < 0) return fail(PA_ERR_ALIAS, "two query rows of the plan map to the same cache slot");
    if (plan->device < 0) return fail(PA_ERR_INVALID_ARGUMENT, "host-only plan: no device to run on");
    int cur = -1;
    PA_CUDA_TRY(cudaGetDevice(&cur));
    if (cur != plan->device)
        return fail(PA_ERR_INVALID_ARGUMENT, "current device %d is not the plan's device %d", cur, plan->device);
    cudaError_t e = pa::launch_append(new_k, new_v, k_cache, v_cache, plan->d_seqs, plan->d_q2seq, plan->d_bt,
                                      plan->table_width, plan->page_size, num_kv_heads, (int32_t)kb, (int32_t)vb,
                                      (int64_t)plan->Nq * num_kv_heads, (cudaStream_t)stream);
    if (e != cudaSuccess) return fail(PA_ERR_CUDA, "append kernel launch failed: %s", cudaGetErrorString(e));
    plan->last_stream = (cudaStream_t)stream;
    plan->last_launches = 1;
    plan->last_kernels = PA_KERNEL_APPEND;
    return ok();
}

// Work lists of the tensor-core backward for one (group size, causal, window), longest first:
// the 128-key tiles of every sequence that some query sees (cost: the rows that see them) for the
// dK/dV kernel, and blocks of at most 128 rows (cost: the keys they see) for the dQ kernel. Key tiles
// that touch a page referenced more than once in the plan (sequences sharing a prefix page, or a
// page listed twice) are "ordered": their rows go to scratch, and the ordered pass's list gives
// every cache row those tiles touch with its scratch rows in (sequence, key) order. One upload; the
// host blob stays with the plan.
static pa_status build_backward_lists(pa_plan* plan, int32_t G, int causal, int32_t window, cudaStream_t st) {
    const int KT = pa::backward_key_tile(), qpb = std::max(1, pa::backward_row_block() / G);
    const int32_t ps = plan->page_size;
    std::vector<int32_t> refs_per_page((size_t)std::max(1, plan->num_pages), 0);
    for (int32_t si = 0; si < plan->S; ++si) {
        const int64_t used = ((int64_t)plan->seqs[si].L + ps - 1) / ps;
        for (int64_t b = 0; b < used; ++b) ++refs_per_page[plan->bt[(size_t)si * plan->table_width + b]];
    }
    auto page_of = [&](int32_t si, int64_t t) { return plan->bt[(size_t)si * plan->table_width + t / ps]; };
    std::vector<std::pair<int64_t, pa::BwdKeyUnit>> ku;
    std::vector<std::pair<int64_t, pa::BwdRowUnit>> ru;
    std::vector<std::pair<int64_t, int32_t>> slot_refs;  // (cache row, scratch row) of ordered tiles
    int32_t n_ord = 0;
    for (int32_t si = 0; si < plan->S; ++si) {
        const pa::SeqInfo& q_ = plan->seqs[si];
        if (q_.n == 0) continue;
        const int64_t base = (int64_t)q_.L - q_.n;  // position of query 0
        for (int64_t k0 = 0; k0 < q_.L; k0 += KT) {
            const int64_t kmax = std::min<int64_t>(k0 + KT, q_.L);
            const int64_t jlo = causal ? std::max<int64_t>(0, k0 - base) : 0;
            const int64_t jhi = window > 0 ? std::min<int64_t>(q_.n, kmax - 1 + window - base) : q_.n;
            if (jhi <= jlo) continue;
            bool shared = false;
            for (int64_t t = k0; t < kmax && !shared; t += std::min<int64_t>(ps - t % ps, kmax - t))
                shared = refs_per_page[page_of(si, t)] > 1;
            int32_t ord = -1;
            if (shared) {
                ord = n_ord++;
                for (int64_t t = k0; t < kmax; ++t)
                    slot_refs.push_back({(int64_t)page_of(si, t) * ps + t % ps, ord * KT + (int32_t)(t - k0)});
            }
            ku.push_back({jhi - jlo, pa::BwdKeyUnit{si, (int32_t)k0, ord, 0}});
        }
        for (int32_t j0 = 0; j0 < q_.n; j0 += qpb) {
            const int32_t j1 = std::min(q_.n, j0 + qpb);
            int32_t lo = 0, hi = 0;
            visible_union(q_.L, q_.n, j0, j1, causal != 0, window, &lo, &hi);
            ru.push_back({(int64_t)hi - lo, pa::BwdRowUnit{si, j0, j1, 0}});
        }
    }
    auto longer = [](const auto& a, const auto& b) { return a.first > b.first; };
    std::stable_sort(ku.begin(), ku.end(), longer);
    std::stable_sort(ru.begin(), ru.end(), longer);
    // ordered pass: group the scratch rows by cache row, keeping (sequence, key) order within a row
    std::stable_sort(slot_refs.begin(), slot_refs.end(),
                     [](const auto& a, const auto& b) { return a.first < b.first; });
    std::vector<pa::BwdSlotSum> sums;
    std::vector<int32_t> refs(slot_refs.size());
    for (size_t i = 0; i < slot_refs.size(); ++i) {
        if (i == 0 || slot_refs[i].first != slot_refs[i - 1].first)
            sums.push_back(pa::BwdSlotSum{slot_refs[i].first, (int32_t)i, 0});
        ++sums.back().count;
        refs[i] = slot_refs[i].second;
    }
    auto align = [](size_t x) { return (x + 255) & ~size_t(255); };
    const size_t row_off = align(ku.size() * sizeof(pa::BwdKeyUnit));
    const size_t sums_off = align(row_off + ru.size() * sizeof(pa::BwdRowUnit));
    const size_t refs_off = align(sums_off + sums.size() * sizeof(pa::BwdSlotSum));
    std::vector<char> blob(std::max<size_t>(16, refs_off + refs.size() * sizeof(int32_t)));
    for (size_t i = 0; i < ku.size(); ++i)
        std::memcpy(blob.data() + i * sizeof(pa::BwdKeyUnit), &ku[i].second, sizeof(pa::BwdKeyUnit));
    for (size_t i = 0; i < ru.size(); ++i)
        std::memcpy(blob.data() + row_off + i * sizeof(pa::BwdRowUnit), &ru[i].second, sizeof(pa::BwdRowUnit));
    if (!sums.empty()) std::memcpy(blob.data() + sums_off, sums.data(), sums.size() * sizeof(pa::BwdSlotSum));
    if (!refs.empty()) std::memcpy(blob.data() + refs_off, refs.data(), refs.size() * sizeof(int32_t));
    // the cached lists are invalid from here until the new ones are uploaded: a failure below
    // leaves the plan to rebuild them on its next call
    plan->bwd_group = 0;
    if (plan->bwd_dev) {
        PA_CUDA_TRY(lib_free(plan->bwd_dev, plan->device, st));
        plan->bwd_dev = nullptr;
    }
    PA_CUDA_TRY(lib_malloc(&plan->bwd_dev, blob.size(), st));
    PA_CUDA_TRY(upload(plan->bwd_dev, blob.data(), blob.size(), st));
    plan->bwd_host.push_back(std::move(blob));
    plan->bwd_group = G;
    plan->bwd_causal = causal;
    plan->bwd_window = window;
    plan->bwd_nkey = (int32_t)ku.size();
    plan->bwd_nrow = (int32_t)ru.size();
    plan->bwd_row_off = row_off;
    plan->bwd_nord = n_ord;
    plan->bwd_nsums = (int32_t)sums.size();
    plan->bwd_sums_off = sums_off;
    plan->bwd_refs_off = refs_off;
    plan->uploaded_bytes += (int64_t)plan->bwd_host.back().size();
    return PA_OK;
}

pa_status pa_backward(pa_plan* plan, const void* q, const void* k_cache, const void* v_cache, const void* out,
                      const float* lse, const void* d_out, pa_dtype dtype, int32_t num_q_heads, int32_t num_kv_heads,
                      int32_t head_dim, int32_t v_head_dim, float scale, int causal, int32_t window, float* d_q,
                      float* d_k_cache, float* d_v_cache, pa_stream stream) {
    if (!plan) return fail(PA_ERR_INVALID_ARGUMENT, "plan is NULL");
    {
        if (dtype != PA_F32 && dtype != PA_BF16 && dtype != PA_F16) return fail(PA_ERR_DTYPE, "unknown dtype %d", (int)dtype);
        if (num_q_heads <= 0 || num_kv_heads <= 0 || num_q_heads % num_kv_heads)
            return fail(PA_ERR_SHAPE, "query heads (%d) must be a positive multiple of kv heads (%d)", num_q_heads, num_kv_heads);
        if (head_dim <= 0 || v_head_dim <= 0) return fail(PA_ERR_SHAPE, "head dims must be positive");
        if (head_dim > 1024 || v_head_dim > 1024) return fail(PA_ERR_UNSUPPORTED, "head dims above 1024 are not supported");
        if (!std::isfinite(scale) || !(scale > 0.0f)) return fail(PA_ERR_INVALID_ARGUMENT, "scale must be finite and > 0");
        if (causal != 0 && causal != 1) return fail(PA_ERR_INVALID_ARGUMENT, "causal must be 0 or 1");
        if (window < 0) return fail(PA_ERR_INVALID_ARGUMENT, "window must be >= 0");
    }
    const int64_t es = (int64_t)dtype_size(dtype);
    const int64_t nq = plan->Nq, pages = plan->num_pages, ps = plan->page_size;
    int64_t n_q, n_k, n_v, n_o, n_l, n_dq, n_dk, n_dv;
    if (!product({nq, num_q_heads, head_dim, es}, &n_q) || !product({pages, ps, num_kv_heads, head_dim, es}, &n_k) ||
        !product({pages, ps, num_kv_heads, v_head_dim, es}, &n_v) || !product({nq, num_q_heads, v_head_dim, es}, &n_o) ||
        !product({nq, num_q_heads, 4}, &n_l) || !product({nq, num_q_heads, head_dim, 4}, &n_dq) ||
        !product({pages, ps, num_kv_heads, head_dim, 4}, &n_dk) || !product({pages, ps, num_kv_heads, v_head_dim, 4}, &n_dv))
        return fail(PA_ERR_BOUNDS, "tensor size overflows 64-bit byte counts");
    if (nq == 0) return ok();
    if (!q || !k_cache || !v_cache || !out || !lse || !d_out || !d_q || !d_k_cache || !d_v_cache)
        return fail(PA_ERR_INVALID_ARGUMENT, "a required pointer is NULL");
    for (const void* ptr : {q, k_cache, v_cache, out, (const void*)lse, d_out, (const void*)d_q, (const void*)d_k_cache,
                            (const void*)d_v_cache})
        if ((uintptr_t)ptr % 16 != 0) return fail(PA_ERR_INVALID_ARGUMENT, "device pointers must be 16-byte aligned");
    auto R = [](const void* p, int64_t n) { return Range{(uintptr_t)p, (uintptr_t)p + (uintptr_t)n}; };
    const Range outs[3] = {R(d_q, n_dq), R(d_k_cache, n_dk), R(d_v_cache, n_dv)};
    const Range ins[6] = {R(q, n_q), R(k_cache, n_k), R(v_cache, n_v), R(out, n_o), R(lse, n_l), R(d_out, n_o)};
    for (int a = 0; a < 3; ++a) {
        for (int b = a + 1; b < 3; ++b)
            if (overlap(outs[a], outs[b])) return fail(PA_ERR_ALIAS, "gradient outputs overlap");
        for (const Range& r : ins)
            if (overlap(outs[a], r)) return fail(PA_ERR_ALIAS, "a gradient output overlaps an input");
    }
    if (plan->device < 0) return fail(PA_ERR_INVALID_ARGUMENT, "host-only plan: no device to run on");
    int cur = -1;
    PA_CUDA_TRY(cudaGetDevice(&cur));
    if (cur != plan->device)
        return fail(PA_ERR_INVALID_ARGUMENT, "current device %d is not the plan's device %d", cur, plan->device);
    const int32_t G = num_q_heads / num_kv_heads;
    cudaStream_t st = (cudaStream_t)stream;
    // The tensor-core kernels index a sequence's rows (queries x G) and the cache rows in 32 bits,
    // load K / V one page box at a time (a page size that divides the 128-key tile or is a multiple
    // of it) and move every operand by TMA (16-byte aligned bases).
    const int64_t cache_rows = (int64_t)plan->num_pages * plan->page_size;
    auto al16 = [](const void* x) { return ((uintptr_t)x & 15u) == 0; };
    const bool tc_layout = plan->page_size % 16 == 0 &&
                           (pa::backward_key_tile() % plan->page_size == 0 ||
                            plan->page_size % pa::backward_key_tile() == 0) &&
                           cache_rows < ((int64_t)1 << 31) && al16(q) && al16(k_cache) && al16(v_cache) &&
                           al16(d_out) && al16(d_k_cache) && al16(d_v_cache);
    if (pa::backward_mma_supported(dtype, head_dim, v_head_dim, G) && tc_layout && nq * (int64_t)G < ((int64_t)1 << 31)) {
        std::lock_guard<std::mutex> lock(plan->mu);
        if (plan->bwd_group != G || plan->bwd_causal != causal || plan->bwd_window != window) {
            pa_status bs = build_backward_lists(plan, G, causal, window, st);
            if (bs != PA_OK) return bs;
        }
        pa_status gs = grow_buffer(&plan->bwd_drow, &plan->bwd_drow_bytes, (size_t)nq * num_q_heads * sizeof(float), st);
        if (gs != PA_OK) return gs;
        const size_t half = (size_t)plan->bwd_nord * num_kv_heads * pa::backward_key_tile() * head_dim;
        if (half > 0) {
            gs = grow_buffer(&plan->bwd_scratch, &plan->bwd_scratch_bytes, 2 * half * sizeof(float), st);
            if (gs != PA_OK) return gs;
        }
        pa::BwdParams2 bp{};
        bp.q = q; bp.k = k_cache; bp.v = v_cache; bp.out = out; bp.lse = lse; bp.dout = d_out;
        bp.drow = plan->bwd_drow; bp.dq = d_q; bp.dk = d_k_cache; bp.dv = d_v_cache;
        bp.seqs = plan->d_seqs; bp.block_tables = plan->d_bt;
        bp.key_units = (const pa::BwdKeyUnit*)plan->bwd_dev;
        bp.row_units = (const pa::BwdRowUnit*)((const char*)plan->bwd_dev + plan->bwd_row_off);
        bp.scratch_k = half > 0 ? plan->bwd_scratch : nullptr;
        bp.scratch_v = half > 0 ? plan->bwd_scratch + half : nullptr;
        bp.slot_sums = (const pa::BwdSlotSum*)((const char*)plan->bwd_dev + plan->bwd_sums_off);
        bp.slot_refs = (const int32_t*)((const char*)plan->bwd_dev + plan->bwd_refs_off);
        bp.table_width = plan->table_width; bp.page_size = plan->page_size;
        bp.hq = num_q_heads; bp.hkv = num_kv_heads; bp.group = G; bp.d = head_dim;
        bp.scale = scale; bp.scale_log2 = scale * 1.4426950408889634f;
        bp.causal = causal; bp.window = window;
        bp.num_pages = plan->num_pages;
        bp.err = plan->d_err;
        cudaError_t e = pa::launch_backward_mma(bp, dtype, plan->bwd_nkey, plan->bwd_nrow, nq * num_q_heads,
                                                plan->bwd_nsums, st);
        if (e != cudaSuccess) return fail(PA_ERR_CUDA, "backward kernel launch failed: %s", cudaGetErrorString(e));
        plan->last_stream = st;
        plan->last_launches = 1 + (plan->bwd_nkey > 0 ? 1 : 0) + (plan->bwd_nrow > 0 ? 1 : 0) + (plan->bwd_nsums > 0 ? 1 : 0);
        plan->last_kernels = PA_KERNEL_BACKWARD_TC;
        return ok();
    }
    cudaError_t e = pa::launch_backward(q, k_cache, v_cache, out, lse, d_out, d_q, d_k_cache, d_v_cache,
                                        plan->d_seqs, plan->d_q2seq, plan->d_bt, plan->table_width, plan->page_size,
                                        num_q_heads, num_kv_heads, head_dim, v_head_dim, scale, causal, window,
                                        nq * num_q_heads, dtype, (cudaStream_t)stream);
    if (e != cudaSuccess) return fail(PA_ERR_CUDA, "backward kernel launch failed: %s", cudaGetErrorString(e));
    plan->last_stream = (cudaStream_t)stream;
    plan->last_launches = 1;
    plan->last_kernels = PA_KERNEL_BACKWARD_SIMT;
    return ok();
}

// Whether some page is used by more than one key of the plan (a shared prefix, a page listed twice).
static bool plan_has_shared_pages(pa_plan* plan) {
    if (plan->shared_pages < 0) {
        std::vector<int32_t> refs((size_t)std::max(1, plan->num_pages), 0);
        bool shared = false;
        for (int32_t si = 0; si < plan->S && !shared; ++si) {
            const int64_t used = ((int64_t)plan->seqs[si].L + plan->page_size - 1) / plan->page_size;
            for (int64_t b = 0; b < used && !shared; ++b)
                shared = ++refs[plan->bt[(size_t)si * plan->table_width + b]] > 1;
        }
        plan->shared_pages = shared ? 1 : 0;
    }
    return plan->shared_pages == 1;
}

// Work lists of the tensor-core MLA backward for one (heads, causal, window): the 128-key tiles of
// every sequence that some of its rows see (each with its columns in the dS' scratch), and one dQ
// unit per sequence with rows, over the same tiles. One upload; the host blob stays with the plan.
static pa_status build_mla_backward_lists(pa_plan* plan, int32_t H, int causal, int32_t window, cudaStream_t st) {
    const int KT = pa::kMlaBwdKeyTile;
    std::vector<pa::MlaKeyTile> tiles;
    std::vector<pa::MlaDqUnit> units;
    int64_t cols = 0;
    for (int32_t si = 0; si < plan->S; ++si) {
        const pa::SeqInfo& q_ = plan->seqs[si];
        if (q_.n == 0) continue;
        // keys any row sees: from the first query's window start to the end of the sequence
        const int64_t first = (int64_t)q_.L - q_.n;
        const int64_t lo = window > 0 ? std::max<int64_t>(0, first - window + 1) : 0;
        const int64_t k0 = lo / KT * KT;
        const int64_t n_t = q_.L > k0 ? (q_.L - k0 + KT - 1) / KT : 0;
        units.push_back({si, (int32_t)k0, (int32_t)(k0 + n_t * KT), (int32_t)cols});
        for (int64_t i = 0; i < n_t; ++i) {
            tiles.push_back({si, (int32_t)(k0 + i * KT), (int32_t)cols, 0});
            cols += KT;
        }
    }
    if (cols > INT32_MAX) return fail(PA_ERR_BOUNDS, "MLA backward scratch too wide");
    (void)causal;
    auto align = [](size_t x) { return (x + 255) & ~size_t(255); };
    const size_t dq_off = align(tiles.size() * sizeof(pa::MlaKeyTile));
    const size_t bytes = std::max<size_t>(256, align(dq_off + units.size() * sizeof(pa::MlaDqUnit)));
    plan->mla_bwd_host.assign(bytes, 0);
    if (!tiles.empty()) std::memcpy(plan->mla_bwd_host.data(), tiles.data(), tiles.size() * sizeof(pa::MlaKeyTile));
    if (!units.empty())
        std::memcpy(plan->mla_bwd_host.data() + dq_off, units.data(), units.size() * sizeof(pa::MlaDqUnit));
    if (plan->mla_bwd_dev) PA_CUDA_TRY(lib_free(plan->mla_bwd_dev, plan->device, st));
    plan->mla_bwd_dev = nullptr;
    plan->mla_bwd_h = 0;
    PA_CUDA_TRY(lib_malloc(&plan->mla_bwd_dev, bytes, st));
    PA_CUDA_TRY(upload(plan->mla_bwd_dev, plan->mla_bwd_host.data(), bytes, st));
    plan->uploaded_bytes += (int64_t)bytes;
    plan->mla_ntiles = (int32_t)tiles.size();
    plan->mla_ndq = (int32_t)units.size();
    plan->mla_dq_off = dq_off;
    plan->mla_ds_cols = std::max<int64_t>(cols, KT);
    plan->mla_bwd_h = H;
    plan->mla_bwd_causal = causal;
    plan->mla_bwd_window = window;
    return PA_OK;
}

pa_status pa_mla_backward(pa_plan* plan, const void* q_latent, const void* q_rope, const void* latent_cache,
                          const void* rope_cache, const void* out, const float* lse, const void* d_out, pa_dtype dtype,
                          int32_t num_heads, int32_t latent_dim, int32_t rope_dim, float scale, int causal,
                          int32_t window, float* d_q_latent, float* d_q_rope, float* d_latent_cache, float* d_rope_cache,
                          pa_stream stream) {
    if (!plan) return fail(PA_ERR_INVALID_ARGUMENT, "plan is NULL");
    if (dtype != PA_F32 && dtype != PA_BF16 && dtype != PA_F16) return fail(PA_ERR_DTYPE, "unknown dtype %d", (int)dtype);
    if (num_heads <= 0) return fail(PA_ERR_SHAPE, "num_heads must be positive");
    if (latent_dim <= 0 || latent_dim > 1024) return fail(PA_ERR_UNSUPPORTED, "latent_dim must be in [1, 1024]");
    if (rope_dim <= 0 || rope_dim > 256) return fail(PA_ERR_UNSUPPORTED, "rope_dim must be in [1, 256]");
    if (!std::isfinite(scale) || !(scale > 0.0f)) return fail(PA_ERR_INVALID_ARGUMENT, "scale must be finite and > 0");
    if (causal != 0 && causal != 1) return fail(PA_ERR_INVALID_ARGUMENT, "causal must be 0 or 1");
    if (window < 0) return fail(PA_ERR_INVALID_ARGUMENT, "window must be >= 0");
    const int64_t es = (int64_t)dtype_size(dtype);
    const int64_t nq = plan->Nq, pages = plan->num_pages, ps = plan->page_size;
    int64_t n_ql, n_qr, n_lat, n_rope, n_o, n_l, n_dql, n_dqr, n_dlat, n_drope;
    if (!product({nq, num_heads, latent_dim, es}, &n_ql) || !product({nq, num_heads, rope_dim, es}, &n_qr) ||
        !product({pages, ps, latent_dim, es}, &n_lat) || !product({pages, ps, rope_dim, es}, &n_rope) ||
        !product({nq, num_heads, latent_dim, es}, &n_o) || !product({nq, num_heads, 4}, &n_l) ||
        !product({nq, num_heads, latent_dim, 4}, &n_dql) || !product({nq, num_heads, rope_dim, 4}, &n_dqr) ||
        !product({pages, ps, latent_dim, 4}, &n_dlat) || !product({pages, ps, rope_dim, 4}, &n_drope))
        return fail(PA_ERR_BOUNDS, "tensor size overflows 64-bit byte counts");
    if (nq == 0) return ok();
    if (!q_latent || !q_rope || !latent_cache || !rope_cache || !out || !lse || !d_out || !d_q_latent || !d_q_rope ||
        !d_latent_cache || !d_rope_cache)
        return fail(PA_ERR_INVALID_ARGUMENT, "a required pointer is NULL");
    for (const void* ptr : {q_latent, q_rope, latent_cache, rope_cache, out, (const void*)lse, d_out,
                            (const void*)d_q_latent, (const void*)d_q_rope, (const void*)d_latent_cache,
                            (const void*)d_rope_cache})
        if ((uintptr_t)ptr % 16 != 0) return fail(PA_ERR_INVALID_ARGUMENT, "device pointers must be 16-byte aligned");
    auto R = [](const void* p, int64_t n) { return Range{(uintptr_t)p, (uintptr_t)p + (uintptr_t)n}; };
    const Range outs[4] = {R(d_q_latent, n_dql), R(d_q_rope, n_dqr), R(d_latent_cache, n_dlat), R(d_rope_cache, n_drope)};
    const Range ins[7] = {R(q_latent, n_ql), R(q_rope, n_qr), R(latent_cache, n_lat), R(rope_cache, n_rope),
                          R(out, n_o), R(lse, n_l), R(d_out, n_o)};
    for (int a = 0; a < 4; ++a) {
        for (int b = a + 1; b < 4; ++b)
            if (overlap(outs[a], outs[b])) return fail(PA_ERR_ALIAS, "gradient outputs overlap");
        for (const Range& r : ins)
            if (overlap(outs[a], r)) return fail(PA_ERR_ALIAS, "a gradient output overlaps an input");
    }
    if (plan->device < 0) return fail(PA_ERR_INVALID_ARGUMENT, "host-only plan: no device to run on");
    int cur = -1;
    PA_CUDA_TRY(cudaGetDevice(&cur));
    if (cur != plan->device)
        return fail(PA_ERR_INVALID_ARGUMENT, "current device %d is not the plan's device %d", cur, plan->device);
    cudaStream_t st = (cudaStream_t)stream;
    // The tensor-core path: bf16 / fp16, latent 512, rope 64, every sequence's rows (queries x heads)
    // within one block of 128, pages of a size the key tiles take whole, no page used twice (each
    // cache row then has one writer), 32-bit cache rows.
    bool tc = pa::mla_backward_tc_supported(dtype, latent_dim, rope_dim, num_heads) && ps % 16 == 0 &&
              (pa::kMlaBwdKeyTile % ps == 0 || ps % pa::kMlaBwdKeyTile == 0) && pages * ps < ((int64_t)1 << 31) &&
              nq * num_heads < ((int64_t)1 << 31);
    for (int32_t si = 0; tc && si < plan->S; ++si) tc = (int64_t)plan->seqs[si].n * num_heads <= 128;
    if (tc) {
        std::lock_guard<std::mutex> lock(plan->mu);
        tc = !plan_has_shared_pages(plan);
        if (tc) {
            if (plan->mla_bwd_h != num_heads || plan->mla_bwd_causal != causal || plan->mla_bwd_window != window) {
                pa_status bs = build_mla_backward_lists(plan, num_heads, causal, window, st);
                if (bs != PA_OK) return bs;
            }
            pa_status gs = grow_buffer(&plan->bwd_drow, &plan->bwd_drow_bytes, (size_t)nq * num_heads * sizeof(float), st);
            if (gs != PA_OK) return gs;
            gs = grow_buffer(&plan->mla_ds, &plan->mla_ds_bytes, (size_t)128 * plan->mla_ds_cols * 2, st);
            if (gs != PA_OK) return gs;
            cudaError_t e = pa::launch_bwd_dot(out, d_out, plan->bwd_drow, nq * num_heads, latent_dim, dtype, st);
            if (e == cudaSuccess) {
                pa::MlaBwdTcParams mp{};
                mp.ql = q_latent; mp.qr = q_rope; mp.lat = latent_cache; mp.rope = rope_cache; mp.dout = d_out;
                mp.lse = lse; mp.drow = plan->bwd_drow;
                mp.dql = d_q_latent; mp.dqr = d_q_rope; mp.dlat = d_latent_cache; mp.drope = d_rope_cache;
                mp.ds = plan->mla_ds; mp.ds_cols = plan->mla_ds_cols;
                mp.seqs = plan->d_seqs; mp.block_tables = plan->d_bt;
                mp.tiles = (const pa::MlaKeyTile*)plan->mla_bwd_dev;
                mp.dq_units = (const pa::MlaDqUnit*)((const char*)plan->mla_bwd_dev + plan->mla_dq_off);
                mp.table_width = plan->table_width; mp.page_size = plan->page_size; mp.h = num_heads;
                mp.num_pages = plan->num_pages;
                mp.scale = scale; mp.scale_log2 = scale * 1.4426950408889634f;
                mp.causal = causal; mp.window = window;
                mp.err = plan->d_err;
                e = pa::launch_mla_backward_tc(mp, dtype, plan->mla_ntiles, plan->mla_ndq, nq, st);
            }
            if (e != cudaSuccess) return fail(PA_ERR_CUDA, "MLA backward kernel launch failed: %s", cudaGetErrorString(e));
            plan->last_stream = st;
            plan->last_launches = 1 + (plan->mla_ntiles > 0 ? 1 : 0) + (plan->mla_ndq > 0 ? 1 : 0);
            plan->last_kernels = PA_KERNEL_BACKWARD_TC;
            return ok();
        }
    }
    cudaError_t e = pa::launch_mla_backward(q_latent, q_rope, latent_cache, rope_cache, out, lse, d_out, d_q_latent,
                                            d_q_rope, d_latent_cache, d_rope_cache, plan->d_seqs, plan->d_q2seq,
                                            plan->d_bt, plan->table_width, plan->page_size, num_heads, latent_dim,
                                            rope_dim, scale, causal, window, nq * num_heads, dtype, (cudaStream_t)stream);
    if (e != cudaSuccess) return fail(PA_ERR_CUDA, "MLA backward kernel launch failed: %s", cudaGetErrorString(e));
    plan->last_stream = (cudaStream_t)stream;
    plan->last_launches = 1;
    plan->last_kernels = PA_KERNEL_BACKWARD_SIMT;
    return ok();
}

pa_status pa_plan_device_status(const pa_plan* plan, int32_t* code) {
    if (!plan || !code) return fail(PA_ERR_INVALID_ARGUMENT, "plan or code is NULL");
    *code = 0;
    if (plan->device < 0) return ok();
    int v = 0;
    PA_CUDA_TRY(cudaMemcpy(&v, plan->d_err, sizeof v, cudaMemcpyDeviceToHost));
    *code = v;
    return ok();
}

const char* pa_status_string(pa_status s) {
    switch (s) {
        case PA_OK: return "PA_OK";
        case PA_ERR_INVALID_ARGUMENT: return "PA_ERR_INVALID_ARGUMENT";
        case PA_ERR_SHAPE: return "PA_ERR_SHAPE";
        case PA_ERR_DTYPE: return "PA_ERR_DTYPE";
        case PA_ERR_BOUNDS: return "PA_ERR_BOUNDS";
        case PA_ERR_ALIAS: return "PA_ERR_ALIAS";
        case PA_ERR_UNSUPPORTED: return "PA_ERR_UNSUPPORTED";
        case PA_ERR_CUDA: return "PA_ERR_CUDA";
    }
    return "PA_ERR_UNKNOWN";
}

const char* pa_last_error_message(void) { return g_msg; }

const char* pa_version(void) { return "0.1.0"; }

}  // extern "C"
