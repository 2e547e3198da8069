// Backward of paged GQA attention on the tensor cores (bf16 / fp16, D == Dv in {64, 128}, G dividing
// 128): the parts around the two tcgen05 kernels of backward_tc.cu, deterministic and free of
// per-key atomics (boostr `standard_attention_bwd`; ruDNN's recompute-based backward, its "ordered"
// history pass in spirit). With P recomputed from Q, K and the forward's lse:
//     P = exp(scale q.k - lse),  dP = dO . v,  dS = P (dP - Drow),  Drow = dO . O
//     dV_k += P dO,   dK_k += scale dS q,   dQ_row += scale dS k
//
//   bwd_dot_kernel     Drow for every (query, head) row (a warp per row).
//   (backward_tc.cu)   dK, dV: key-major, each key's rows summed by one CTA.
//   bwd_ordered_kernel the ordered pass: a warp per cache row of a page the plan references more
//                      than once sums the scratch rows that map to it in sequence order and adds
//                      the sum once, so shared pages give the same bits on every run.
//   (backward_tc.cu)   dQ: query-major, each 128-row block's dQ summed in TMEM and written once.
#include <mutex>

#include "device_common.cuh"
#include "pa_internal.h"

namespace pa {

// ---- Drow = dO . O per (query, head) row ----------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(128) bwd_dot_kernel(const T* __restrict__ out, const T* __restrict__ dout,
                                                      float* __restrict__ drow, int64_t rows, int dv) {
    const int64_t row = (int64_t)blockIdx.x * 4 + (threadIdx.x >> 5);
    if (row >= rows) return;
    const int lane = threadIdx.x & 31;
    float acc = 0.f;
    for (int c = lane; c < dv; c += 32) acc += to_f32(out[row * dv + c]) * to_f32(dout[row * dv + c]);
    acc = warp_sum(acc);
    if (lane == 0) drow[row] = acc;
}

// ---- ordered pass: a warp per (shared cache row, KV head) -------------------------------------
// refs encode (scratch tile, row) as tile * kt + row; scratch rows are [tile][Hkv][kt][D].
template <int D>
__global__ void __launch_bounds__(128) bwd_ordered_kernel(const BwdParams2 p, int num_sums, int kt) {
    const int item = blockIdx.x * 4 + (threadIdx.x >> 5);
    if (item >= num_sums) return;
    const int lane = threadIdx.x & 31, kvh = blockIdx.y;
    const BwdSlotSum w = p.slot_sums[item];
    const int64_t dst = (w.slot * p.hkv + kvh) * D;
    for (int d = lane * 2; d < D; d += 64) {
        float2 ak = make_float2(0.f, 0.f), av = ak;
        for (int i = 0; i < w.count; ++i) {  // in the order the host listed: by sequence, then key
            const int32_t ref = p.slot_refs[w.begin + i];
            const int64_t src = (((int64_t)(ref / kt) * p.hkv + kvh) * kt + ref % kt) * D + d;
            const float2 k2 = *reinterpret_cast<const float2*>(p.scratch_k + src);
            const float2 v2 = *reinterpret_cast<const float2*>(p.scratch_v + src);
            ak.x += k2.x; ak.y += k2.y;
            av.x += v2.x; av.y += v2.y;
        }
        // the only writer of this row: one add onto the caller's (zeroed) cache
        p.dk[dst + d] += ak.x; p.dk[dst + d + 1] += ak.y;
        p.dv[dst + d] += av.x; p.dv[dst + d + 1] += av.y;
    }
}

// ---------------------------------------------------------------------------------------------
std::mutex& side_mutex() {
    static std::mutex m;
    return m;
}

// Called with side_mutex() held. Created on first use per device, kept for the process's life.
cudaError_t side_stream(SideStream** out) {
    static SideStream per_device[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    SideStream& s = per_device[dev];
    if (!s.stream) {
        e = cudaStreamCreateWithFlags(&s.stream, cudaStreamNonBlocking);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&s.fork, cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&s.join, cudaEventDisableTiming);
        if (e != cudaSuccess) {
            if (s.fork) cudaEventDestroy(s.fork);
            if (s.stream) cudaStreamDestroy(s.stream);
            s = SideStream{};
            return e;
        }
    }
    *out = &s;
    return cudaSuccess;
}

namespace {

template <typename T, int D>
cudaError_t bwd_launch_d(const BwdParams2& p, int num_key_units, int num_row_units, int64_t rows, int num_sums,
                         cudaStream_t st) {
    cudaError_t e;
    bwd_dot_kernel<T><<<(unsigned)((rows + 3) / 4), 128, 0, st>>>(static_cast<const T*>(p.out),
                                                                   static_cast<const T*>(p.dout), p.drow, rows, D);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    // dQ on a side stream and dK/dV (then the ordered pass) on the caller's stream, so that each
    // kernel's CTAs fill the SMs the other one's last wave leaves idle; both only read what the
    // Drow kernel and the caller wrote. dQ is issued first (its CTAs start first; measured about
    // 2 % faster than the other order). The side stream forks from and joins back into the
    // caller's stream through events, so the call stays stream-ordered (and capturable).
    const bool fork = num_key_units > 0 && num_row_units > 0;
    std::unique_lock<std::mutex> lk(side_mutex(), std::defer_lock);
    SideStream* side = nullptr;
    if (fork) {
        lk.lock();  // one fork/join at a time: each wait pairs with its own record
        e = side_stream(&side);
        if (e != cudaSuccess) return e;
        e = cudaEventRecord(side->fork, st);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(side->stream, side->fork, 0);
        if (e != cudaSuccess) return e;
    }
    if (num_row_units > 0)
        e = launch_backward_tc_dq(p, std::is_same<T, __nv_bfloat16>::value ? PA_BF16 : PA_F16, num_row_units,
                                  rows / p.hq, fork ? side->stream : st);
    if (e == cudaSuccess && num_key_units > 0)
        e = launch_backward_tc_dkdv(p, std::is_same<T, __nv_bfloat16>::value ? PA_BF16 : PA_F16, num_key_units,
                                    rows / p.hq, st);
    if (e == cudaSuccess && num_sums > 0) {
        bwd_ordered_kernel<D><<<dim3((num_sums + 3) / 4, p.hkv), 128, 0, st>>>(p, num_sums, backward_tc_key_tile());
        e = cudaGetLastError();
    }
    if (fork) {  // joined on every path, so that a capture on the caller's stream never ends unjoined
        cudaError_t j = cudaEventRecord(side->join, side->stream);
        if (j == cudaSuccess) j = cudaStreamWaitEvent(st, side->join, 0);
        if (e == cudaSuccess) e = j;
    }
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd_dot(const void* out, const void* dout, float* drow, int64_t rows, int dv, pa_dtype dt,
                           cudaStream_t st) {
    if (rows == 0) return cudaSuccess;
    const unsigned grid = (unsigned)((rows + 3) / 4);
    if (dt == PA_BF16)
        bwd_dot_kernel<__nv_bfloat16><<<grid, 128, 0, st>>>(static_cast<const __nv_bfloat16*>(out),
                                                             static_cast<const __nv_bfloat16*>(dout), drow, rows, dv);
    else
        bwd_dot_kernel<__half><<<grid, 128, 0, st>>>(static_cast<const __half*>(out), static_cast<const __half*>(dout),
                                                      drow, rows, dv);
    return cudaGetLastError();
}

bool backward_mma_supported(pa_dtype dt, int d, int dv, int group) {
    // both tcgen05 passes walk 128-row blocks: 128 / G queries x the G heads of a KV head
    return (dt == PA_BF16 || dt == PA_F16) && d == dv && (d == 64 || d == 128) && group >= 1 && 128 % group == 0;
}

int backward_key_tile() { return backward_tc_key_tile(); }
int backward_row_block() { return backward_tc_row_block(); }

cudaError_t launch_backward_mma(const BwdParams2& p, pa_dtype dt, int num_key_units, int num_row_units, int64_t rows,
                                int num_sums, cudaStream_t st) {
    if (rows == 0) return cudaSuccess;
    if (dt == PA_BF16)
        return p.d == 64 ? bwd_launch_d<__nv_bfloat16, 64>(p, num_key_units, num_row_units, rows, num_sums, st)
                         : bwd_launch_d<__nv_bfloat16, 128>(p, num_key_units, num_row_units, rows, num_sums, st);
    return p.d == 64 ? bwd_launch_d<__half, 64>(p, num_key_units, num_row_units, rows, num_sums, st)
                     : bwd_launch_d<__half, 128>(p, num_key_units, num_row_units, rows, num_sums, st);
}

}  // namespace pa
