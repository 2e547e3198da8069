// End-to-end decode loop through the public C ABI with host buffers, for bench.py's `e2e` figure:
// the loop a serving engine with asynchronous scheduling runs, written in C so that the host side
// costs what the library and the CUDA runtime cost, not an interpreter's dispatch.
//
// Per step: a new plan (pa_plan_create + pa_plan_prepare, their uploads on an upload stream), the
// step's queries copied in from page-locked host memory (upload stream), pa_forward (the caller's
// stream), out and lse copied back into page-locked host memory (download stream), the plan
// released. Two steps are in flight: step i+1's plan and query upload overlap step i's attention,
// step i's download overlaps step i+1's; the host waits for step i's result before it issues step
// i+2. Device and host buffers are double-buffered (index i & 1) so that no copy touches a buffer a
// running step uses. The host buffers are allocated here (page-locked by this runtime) when the
// loop is set up, outside any timed region.
#include <chrono>
#include <cstring>

#include <cuda_runtime.h>
#include <stdint.h>

#include "pa.h"

namespace {

struct E2eLoop {
    // schedule and attention arguments
    const int32_t *seq_lens, *query_offsets, *block_tables;
    int32_t num_seqs, table_width, page_size, num_pages;
    int device;
    const void *k_cache, *v_cache;
    pa_dtype dtype;
    int32_t hq, hkv, d, dv;
    float scale;
    int causal;
    int32_t window;
    // buffers: device ones belong to the caller, host ones to the loop
    void* q_dev[2];
    void* out_dev[2];
    float* lse_dev[2];
    size_t q_bytes, out_bytes, lse_bytes;
    void* q_host = nullptr;
    void* out_host[2] = {};
    float* lse_host[2] = {};
    cudaStream_t up = nullptr, down = nullptr;
    cudaEvent_t h2d[2] = {}, fwd[2] = {}, d2h[2] = {}, ready[2] = {};
    cudaEvent_t fs[4] = {}, fe[4] = {};  // timing: start / end of step i's forward on the compute stream, ring of 4
    long long uploaded = 0;
    double host_us[6] = {};  // plan create, plan prepare, copies, forward, release, waits
    double gpu_us[2] = {};   // device time of the forward kernels, compute stream idle before them

    ~E2eLoop() {
        for (int b = 0; b < 2; ++b) {
            if (h2d[b]) cudaEventDestroy(h2d[b]);
            if (fwd[b]) cudaEventDestroy(fwd[b]);
            if (d2h[b]) cudaEventDestroy(d2h[b]);
            if (ready[b]) cudaEventDestroy(ready[b]);
            for (int r = 2 * b; r < 2 * b + 2; ++r) {
                if (fs[r]) cudaEventDestroy(fs[r]);
                if (fe[r]) cudaEventDestroy(fe[r]);
            }
            if (out_host[b]) cudaFreeHost(out_host[b]);
            if (lse_host[b]) cudaFreeHost(lse_host[b]);
        }
        if (q_host) cudaFreeHost(q_host);
        if (up) cudaStreamDestroy(up);
        if (down) cudaStreamDestroy(down);
    }
};

double since_us(std::chrono::steady_clock::time_point t0) {
    return std::chrono::duration<double, std::micro>(std::chrono::steady_clock::now() - t0).count();
}

}  // namespace

extern "C" {

// Sets up a loop: copies the step's queries (q, host memory, q_bytes) into page-locked memory,
// allocates the page-locked out / lse buffers, the two copy streams and the events. The schedule
// arrays, caches and device buffers must outlive the loop. Returns NULL on a runtime failure.
void* pa_e2e_create(const int32_t* seq_lens, const int32_t* query_offsets, int32_t num_seqs,
                    const int32_t* block_tables, int32_t table_width, int32_t page_size, int32_t num_pages,
                    int device, const void* q, size_t q_bytes, void* const* q_dev, const void* k_cache,
                    const void* v_cache, int dtype, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                    int32_t v_head_dim, float scale, int causal, int32_t window, void* const* out_dev,
                    float* const* lse_dev, size_t out_bytes, size_t lse_bytes) {
    E2eLoop* L = new E2eLoop();
    L->seq_lens = seq_lens; L->query_offsets = query_offsets; L->block_tables = block_tables;
    L->num_seqs = num_seqs; L->table_width = table_width; L->page_size = page_size; L->num_pages = num_pages;
    L->device = device; L->k_cache = k_cache; L->v_cache = v_cache; L->dtype = static_cast<pa_dtype>(dtype);
    L->hq = num_q_heads; L->hkv = num_kv_heads; L->d = head_dim; L->dv = v_head_dim;
    L->scale = scale; L->causal = causal; L->window = window;
    L->q_bytes = q_bytes; L->out_bytes = out_bytes; L->lse_bytes = lse_bytes;
    cudaError_t e = cudaSetDevice(device);
    for (int b = 0; b < 2; ++b) {
        L->q_dev[b] = q_dev[b];
        L->out_dev[b] = out_dev[b];
        L->lse_dev[b] = lse_dev[b];
    }
    if (e == cudaSuccess) e = cudaMallocHost(&L->q_host, q_bytes);
    if (e == cudaSuccess) std::memcpy(L->q_host, q, q_bytes);
    for (int b = 0; b < 2 && e == cudaSuccess; ++b) {
        e = cudaMallocHost(&L->out_host[b], out_bytes);
        if (e == cudaSuccess) e = cudaMallocHost(reinterpret_cast<void**>(&L->lse_host[b]), lse_bytes);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&L->h2d[b], cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&L->fwd[b], cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&L->d2h[b], cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&L->ready[b], cudaEventDisableTiming);
    }
    for (int r = 0; r < 4 && e == cudaSuccess; ++r) {
        e = cudaEventCreate(&L->fs[r]);
        if (e == cudaSuccess) e = cudaEventCreate(&L->fe[r]);
    }
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&L->up, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&L->down, cudaStreamNonBlocking);
    if (e != cudaSuccess) {
        delete L;
        return nullptr;
    }
    return L;
}

void pa_e2e_destroy(void* loop) { delete static_cast<E2eLoop*>(loop); }

// Bytes one step's plan uploaded (schedule and work list), and the host time the steps of the last
// pa_e2e_run spent in each part (microseconds, summed over the steps).
long long pa_e2e_uploaded_bytes(const void* loop) { return static_cast<const E2eLoop*>(loop)->uploaded; }
void pa_e2e_host_times(const void* loop, double* us6) {
    for (int i = 0; i < 6; ++i) us6[i] = static_cast<const E2eLoop*>(loop)->host_us[i];
}
// Device time of the forwards of the last run (summed over its steps but the last) and the time the
// compute stream sat idle before each of them (from the end of the previous step's forward).
void pa_e2e_gpu_times(const void* loop, double* us2) {
    for (int i = 0; i < 2; ++i) us2[i] = static_cast<const E2eLoop*>(loop)->gpu_us[i];
}

// Runs `steps` steps on `stream` (the compute stream) and returns once every step's result is on
// the host. Returns 0, a pa_status (> 0) from a library call, or -(cudaError_t) from a runtime call.
int pa_e2e_run(void* loop, int steps, void* stream) {
    E2eLoop& L = *static_cast<E2eLoop*>(loop);
    if (steps <= 0) return 0;
    cudaStream_t main = static_cast<cudaStream_t>(stream);
    for (double& t : L.host_us) t = 0.0;
    for (double& t : L.gpu_us) t = 0.0;
    pa_plan* cur = nullptr;
    pa_plan* nxt = nullptr;
    int rc = 0;
    auto pa_ok = [&](pa_status s) {
        if (s != PA_OK && rc == 0) rc = (int)s;
        return s == PA_OK;
    };
    auto cu_ok = [&](cudaError_t c) {
        if (c != cudaSuccess && rc == 0) rc = -(int)c;
        return c == cudaSuccess;
    };
    // plan of step j, its uploads on the upload stream, marked by ready[j & 1]
    auto make_plan = [&](int j, pa_plan** p) {
        auto t0 = std::chrono::steady_clock::now();
        bool ok = pa_ok(pa_plan_create(L.seq_lens, L.query_offsets, L.num_seqs, L.block_tables, L.table_width,
                                       L.page_size, L.num_pages, L.device, L.up, p));
        L.host_us[0] += since_us(t0);
        t0 = std::chrono::steady_clock::now();
        ok = ok && pa_ok(pa_plan_prepare(*p, 0, L.dtype, L.hq, L.hkv, L.d, L.dv, L.causal, L.window, L.up, nullptr));
        ok = ok && cu_ok(cudaEventRecord(L.ready[j & 1], L.up));
        L.host_us[1] += since_us(t0);
        return ok;
    };
    bool ok = make_plan(0, &cur);
    for (int i = 0; ok && i < steps; ++i) {
        const int b = i & 1;
        auto t0 = std::chrono::steady_clock::now();
        if (i >= 2) ok = cu_ok(cudaStreamWaitEvent(L.up, L.fwd[b], 0));  // step i-2 has read q_dev[b]
        ok = ok && cu_ok(cudaMemcpyAsync(L.q_dev[b], L.q_host, L.q_bytes, cudaMemcpyHostToDevice, L.up));
        ok = ok && cu_ok(cudaEventRecord(L.h2d[b], L.up));
        ok = ok && cu_ok(cudaStreamWaitEvent(main, L.h2d[b], 0));
        ok = ok && cu_ok(cudaStreamWaitEvent(main, L.ready[b], 0));  // the plan's uploads
        L.host_us[2] += since_us(t0);
        t0 = std::chrono::steady_clock::now();
        ok = ok && cu_ok(cudaEventRecord(L.fs[i & 3], main));
        ok = ok && pa_ok(pa_forward(cur, L.q_dev[b], L.k_cache, L.v_cache, L.dtype, L.hq, L.hkv, L.d, L.dv, L.scale,
                                    L.causal, L.window, L.out_dev[b], L.lse_dev[b], main));
        ok = ok && cu_ok(cudaEventRecord(L.fe[i & 3], main));
        ok = ok && cu_ok(cudaEventRecord(L.fwd[b], main));
        L.host_us[3] += since_us(t0);
        t0 = std::chrono::steady_clock::now();
        ok = ok && cu_ok(cudaStreamWaitEvent(L.down, L.fwd[b], 0));
        ok = ok && cu_ok(cudaMemcpyAsync(L.out_host[b], L.out_dev[b], L.out_bytes, cudaMemcpyDeviceToHost, L.down));
        ok = ok && cu_ok(cudaMemcpyAsync(L.lse_host[b], L.lse_dev[b], L.lse_bytes, cudaMemcpyDeviceToHost, L.down));
        ok = ok && cu_ok(cudaEventRecord(L.d2h[b], L.down));
        L.host_us[2] += since_us(t0);
        if (ok && i + 1 < steps) ok = make_plan(i + 1, &nxt);
        t0 = std::chrono::steady_clock::now();
        pa_plan_info info;
        if (pa_plan_get_info(cur, &info) == PA_OK) L.uploaded = info.uploaded_bytes;
        pa_plan* done = cur;
        cur = nullptr;
        ok = pa_ok(pa_plan_destroy(done)) && ok;  // frees ordered on the compute stream after the step
        L.host_us[4] += since_us(t0);
        t0 = std::chrono::steady_clock::now();
        if (ok && i >= 1) ok = cu_ok(cudaEventSynchronize(L.d2h[b ^ 1]));  // step i-1's result is on the host
        L.host_us[5] += since_us(t0);
        if (ok && i >= 1) {
            float ms = 0.f;
            if (cudaEventElapsedTime(&ms, L.fs[(i - 1) & 3], L.fe[(i - 1) & 3]) == cudaSuccess) L.gpu_us[0] += 1e3 * ms;
            if (i >= 2 && cudaEventElapsedTime(&ms, L.fe[(i - 2) & 3], L.fs[(i - 1) & 3]) == cudaSuccess)
                L.gpu_us[1] += 1e3 * ms;
        }
        cur = nxt;
        nxt = nullptr;
    }
    if (cur) pa_plan_destroy(cur);
    if (nxt) pa_plan_destroy(nxt);
    cu_ok(cudaStreamSynchronize(L.up));
    cu_ok(cudaStreamSynchronize(L.down));
    return rc;
}

}  // extern "C"
