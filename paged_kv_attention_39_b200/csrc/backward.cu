// Backward of paged GQA and MLA attention on the CUDA cores (boostr `standard_attention_bwd`;
// ruDNN's recompute-based backward with float32 atomics). With P recomputed from Q, K and the forward's lse,
//     dV_t += P_t dO,  dP_t = dO . V_t,  D = dO . O,  dS_t = P_t (dP_t - D),
//     dQ = scale * sum_t dS_t K_t,  dK_t += scale * dS_t Q.
// One warp owns one (query, query head) row and walks its visible keys; dQ is accumulated in
// registers and written once, dK/dV are added into the float32 gradient caches with atomics
// (the G heads of a group, every query that sees a key, and sequences sharing a page all add
// into the same slot).
#include "device_common.cuh"

namespace pa {

struct BwdParams {
    const void* q;      // [Nq, Hq, D]
    const void* k;      // [P, ps, Hkv, D]
    const void* v;      // [P, ps, Hkv, Dv]
    const void* out;    // [Nq, Hq, Dv] forward output
    const float* lse;   // [Nq, Hq] forward logsumexp (natural log)
    const void* dout;   // [Nq, Hq, Dv]
    float* dq;          // [Nq, Hq, D] written
    float* dk;          // [P, ps, Hkv, D] accumulated
    float* dv;          // [P, ps, Hkv, Dv] accumulated
    const SeqInfo* seqs;
    const int32_t* q2seq;
    const int32_t* block_tables;
    int32_t table_width, page_size, hq, hkv, group, d, dv_dim, causal, window;
    float scale;
    int64_t rows;
};

template <typename T, int PL>
__global__ void __launch_bounds__(128) backward_kernel(const BwdParams p) {
    const int64_t row = (int64_t)blockIdx.x * 4 + (threadIdx.x >> 5);
    if (row >= p.rows) return;
    const int lane = threadIdx.x & 31;
    const int64_t qi = row / p.hq;
    const int h = (int)(row % p.hq);
    const int kvh = h / p.group;
    const int32_t s = p.q2seq[qi];
    const SeqInfo si = p.seqs[s];
    const int64_t pos = (int64_t)si.L - si.n + (qi - si.q_start);
    const T* qp = static_cast<const T*>(p.q) + row * p.d;
    const T* op = static_cast<const T*>(p.out) + row * p.dv_dim;
    const T* gp = static_cast<const T*>(p.dout) + row * p.dv_dim;
    float qv[PL], gv[PL], dqv[PL];
    float dsum = 0.f;
#pragma unroll
    for (int i = 0; i < PL; ++i) {
        const int c = lane + 32 * i;
        qv[i] = c < p.d ? to_f32(qp[c]) : 0.f;
        gv[i] = c < p.dv_dim ? to_f32(gp[c]) : 0.f;
        dqv[i] = 0.f;
        if (c < p.dv_dim) dsum += gv[i] * to_f32(op[c]);
    }
    const float Drow = warp_sum(dsum);
    const float lse = p.lse[row];
    const int64_t lo = p.window > 0 ? max64(0, pos - p.window + 1) : 0;
    const int64_t hi = p.causal ? pos + 1 : si.L;
    const T* kc = static_cast<const T*>(p.k);
    const T* vc = static_cast<const T*>(p.v);
    const int32_t* bt = p.block_tables + (int64_t)s * p.table_width;
    if (lse != neg_inf()) {
        for (int64_t t = lo; t < hi; ++t) {
            const int64_t slot = (int64_t)bt[t / p.page_size] * p.page_size + t % p.page_size;
            const int64_t kr = (slot * p.hkv + kvh) * p.d;
            const int64_t vr = (slot * p.hkv + kvh) * p.dv_dim;
            float sd = 0.f, pd = 0.f;
            float kv[PL];
#pragma unroll
            for (int i = 0; i < PL; ++i) {
                const int c = lane + 32 * i;
                kv[i] = c < p.d ? to_f32(kc[kr + c]) : 0.f;
                sd += qv[i] * kv[i];
                if (c < p.dv_dim) pd += gv[i] * to_f32(vc[vr + c]);
            }
            const float score = warp_sum(sd) * p.scale;
            const float dp = warp_sum(pd);
            const float pr = __expf(score - lse);
            const float ds = pr * (dp - Drow) * p.scale;
#pragma unroll
            for (int i = 0; i < PL; ++i) {
                const int c = lane + 32 * i;
                if (c < p.d) {
                    dqv[i] += ds * kv[i];
                    atomicAdd(p.dk + kr + c, ds * qv[i]);
                }
                if (c < p.dv_dim) atomicAdd(p.dv + vr + c, pr * gv[i]);
            }
        }
    }
#pragma unroll
    for (int i = 0; i < PL; ++i) {
        const int c = lane + 32 * i;
        if (c < p.d) p.dq[row * p.d + c] = dqv[i];
    }
}

// ---- MLA: the latent is key and value, the rope rows extend the key -----------------------------
struct MlaBwdParams {
    const void* ql;     // [Nq, H, R]
    const void* qr;     // [Nq, H, Pr]
    const void* lat;    // [P, ps, 1, R]
    const void* rope;   // [P, ps, 1, Pr]
    const void* out;    // [Nq, H, R]
    const float* lse;   // [Nq, H]
    const void* dout;   // [Nq, H, R]
    float* dql;         // [Nq, H, R] written
    float* dqr;         // [Nq, H, Pr] written
    float* dlat;        // [P, ps, 1, R] accumulated
    float* drope;       // [P, ps, 1, Pr] accumulated
    const SeqInfo* seqs;
    const int32_t* q2seq;
    const int32_t* block_tables;
    int32_t table_width, page_size, h, r, pr, causal, window;
    float scale;
    int64_t rows;
};

// One warp owns one (query, head) row: lanes hold 32-strided columns of the latent (PL per lane)
// and of the rope part (PR per lane).
template <typename T, int PL, int PR>
__global__ void __launch_bounds__(128) mla_backward_kernel(const MlaBwdParams p) {
    const int64_t row = (int64_t)blockIdx.x * 4 + (threadIdx.x >> 5);
    if (row >= p.rows) return;
    const int lane = threadIdx.x & 31;
    const int64_t qi = row / p.h;
    const int32_t s = p.q2seq[qi];
    const SeqInfo si = p.seqs[s];
    const int64_t pos = (int64_t)si.L - si.n + (qi - si.q_start);
    const T* qlp = static_cast<const T*>(p.ql) + row * p.r;
    const T* qrp = static_cast<const T*>(p.qr) + row * p.pr;
    const T* op = static_cast<const T*>(p.out) + row * p.r;
    const T* gp = static_cast<const T*>(p.dout) + row * p.r;
    float ql[PL], gv[PL], dql[PL], qr[PR], dqr[PR];
    float dsum = 0.f;
#pragma unroll
    for (int i = 0; i < PL; ++i) {
        const int c = lane + 32 * i;
        const bool in = c < p.r;
        ql[i] = in ? to_f32(qlp[c]) : 0.f;
        gv[i] = in ? to_f32(gp[c]) : 0.f;
        dql[i] = 0.f;
        if (in) dsum += gv[i] * to_f32(op[c]);
    }
#pragma unroll
    for (int i = 0; i < PR; ++i) {
        const int c = lane + 32 * i;
        qr[i] = c < p.pr ? to_f32(qrp[c]) : 0.f;
        dqr[i] = 0.f;
    }
    const float Drow = warp_sum(dsum);
    const float lse = p.lse[row];
    const int64_t lo = p.window > 0 ? max64(0, pos - p.window + 1) : 0;
    const int64_t hi = p.causal ? pos + 1 : si.L;
    const T* lc = static_cast<const T*>(p.lat);
    const T* rc = static_cast<const T*>(p.rope);
    const int32_t* bt = p.block_tables + (int64_t)s * p.table_width;
    if (lse != neg_inf()) {
        for (int64_t t = lo; t < hi; ++t) {
            const int64_t slot = (int64_t)bt[t / p.page_size] * p.page_size + t % p.page_size;
            const int64_t lr = slot * p.r, rr = slot * p.pr;
            float sd = 0.f, pd = 0.f;
            float lv[PL], rv[PR];
#pragma unroll
            for (int i = 0; i < PL; ++i) {
                const int c = lane + 32 * i;
                lv[i] = c < p.r ? to_f32(lc[lr + c]) : 0.f;
                sd += ql[i] * lv[i];
                pd += gv[i] * lv[i];
            }
#pragma unroll
            for (int i = 0; i < PR; ++i) {
                const int c = lane + 32 * i;
                rv[i] = c < p.pr ? to_f32(rc[rr + c]) : 0.f;
                sd += qr[i] * rv[i];
            }
            const float score = warp_sum(sd) * p.scale;
            const float dp = warp_sum(pd);
            const float pr = __expf(score - lse);
            const float ds = pr * (dp - Drow) * p.scale;
#pragma unroll
            for (int i = 0; i < PL; ++i) {
                const int c = lane + 32 * i;
                if (c < p.r) {
                    dql[i] += ds * lv[i];
                    atomicAdd(p.dlat + lr + c, ds * ql[i] + pr * gv[i]);
                }
            }
#pragma unroll
            for (int i = 0; i < PR; ++i) {
                const int c = lane + 32 * i;
                if (c < p.pr) {
                    dqr[i] += ds * rv[i];
                    atomicAdd(p.drope + rr + c, ds * qr[i]);
                }
            }
        }
    }
#pragma unroll
    for (int i = 0; i < PL; ++i) {
        const int c = lane + 32 * i;
        if (c < p.r) p.dql[row * p.r + c] = dql[i];
    }
#pragma unroll
    for (int i = 0; i < PR; ++i) {
        const int c = lane + 32 * i;
        if (c < p.pr) p.dqr[row * p.pr + c] = dqr[i];
    }
}

template <typename T, int PL>
static cudaError_t mla_bwd_launch_pr(const MlaBwdParams& p, cudaStream_t st) {
    const unsigned blocks = (unsigned)((p.rows + 3) / 4);
    if (p.pr <= 32) mla_backward_kernel<T, PL, 1><<<blocks, 128, 0, st>>>(p);
    else if (p.pr <= 64) mla_backward_kernel<T, PL, 2><<<blocks, 128, 0, st>>>(p);
    else if (p.pr <= 128) mla_backward_kernel<T, PL, 4><<<blocks, 128, 0, st>>>(p);
    else mla_backward_kernel<T, PL, 8><<<blocks, 128, 0, st>>>(p);
    return cudaGetLastError();
}

template <typename T>
static cudaError_t mla_bwd_launch_t(const MlaBwdParams& p, cudaStream_t st) {
    if (p.r <= 32) return mla_bwd_launch_pr<T, 1>(p, st);
    if (p.r <= 64) return mla_bwd_launch_pr<T, 2>(p, st);
    if (p.r <= 128) return mla_bwd_launch_pr<T, 4>(p, st);
    if (p.r <= 256) return mla_bwd_launch_pr<T, 8>(p, st);
    if (p.r <= 512) return mla_bwd_launch_pr<T, 16>(p, st);
    return mla_bwd_launch_pr<T, 32>(p, st);
}

cudaError_t launch_mla_backward(const void* ql, const void* qr, const void* lat, const void* rope, const void* out,
                                const float* lse, const void* dout, float* dql, float* dqr, float* dlat, float* drope,
                                const SeqInfo* seqs, const int32_t* q2seq, const int32_t* block_tables,
                                int32_t table_width, int32_t page_size, int32_t h, int32_t r, int32_t pr, float scale,
                                int causal, int32_t window, int64_t rows, pa_dtype dt, cudaStream_t st) {
    if (rows == 0) return cudaSuccess;
    MlaBwdParams p{ql, qr, lat, rope, out, lse, dout, dql, dqr, dlat, drope, seqs, q2seq, block_tables, table_width,
                   page_size, h, r, pr, causal, window, scale, rows};
    switch (dt) {
        case PA_F32: return mla_bwd_launch_t<float>(p, st);
        case PA_BF16: return mla_bwd_launch_t<__nv_bfloat16>(p, st);
        default: return mla_bwd_launch_t<__half>(p, st);
    }
}

template <typename T>
static cudaError_t bwd_launch_t(const BwdParams& p, cudaStream_t st) {
    const int widest = max(p.d, p.dv_dim);
    const unsigned blocks = (unsigned)((p.rows + 3) / 4);
    if (widest <= 32) backward_kernel<T, 1><<<blocks, 128, 0, st>>>(p);
    else if (widest <= 64) backward_kernel<T, 2><<<blocks, 128, 0, st>>>(p);
    else if (widest <= 128) backward_kernel<T, 4><<<blocks, 128, 0, st>>>(p);
    else if (widest <= 256) backward_kernel<T, 8><<<blocks, 128, 0, st>>>(p);
    else if (widest <= 512) backward_kernel<T, 16><<<blocks, 128, 0, st>>>(p);
    else backward_kernel<T, 32><<<blocks, 128, 0, st>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_backward(const void* q, const void* k, const void* v, const void* out, const float* lse,
                            const void* dout, float* dq, float* dk, float* dv, const SeqInfo* seqs, const int32_t* q2seq,
                            const int32_t* block_tables, int32_t table_width, int32_t page_size, int32_t hq,
                            int32_t hkv, int32_t d, int32_t dv_dim, float scale, int causal, int32_t window,
                            int64_t rows, pa_dtype dt, cudaStream_t st) {
    if (rows == 0) return cudaSuccess;
    BwdParams p{q, k, v, out, lse, dout, dq, dk, dv, seqs, q2seq, block_tables, table_width, page_size, hq, hkv,
                hq / hkv, d, dv_dim, causal, window, scale, rows};
    switch (dt) {
        case PA_F32: return bwd_launch_t<float>(p, st);
        case PA_BF16: return bwd_launch_t<__nv_bfloat16>(p, st);
        default: return bwd_launch_t<__half>(p, st);
    }
}

}  // namespace pa
