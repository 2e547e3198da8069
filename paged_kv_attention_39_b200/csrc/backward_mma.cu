// Backward of paged GQA attention on the tensor cores (bf16 / fp16, D == Dv in {64, 128}, G dividing
// 128 and at most 16): the parts around the tcgen05 dK/dV kernel (backward_tc.cu), deterministic
// and free of per-key atomics (boostr `standard_attention_bwd`; ruDNN's recompute-based backward,
// its "ordered" history pass in spirit). With P recomputed from Q, K and the forward's lse:
//     P = exp(scale q.k - lse),  dP = dO . v,  dS = P (dP - Drow),  Drow = dO . O
//     dV_k += P dO,   dK_k += scale dS q,   dQ_row += scale dS k
//
//   bwd_dot_kernel     Drow for every (query, head) row (a warp per row).
//   (backward_tc.cu)   dK, dV: key-major on tcgen05, each key's rows summed by one CTA.
//   bwd_ordered_kernel the ordered pass: a warp per cache row of a page the plan references more
//                      than once sums the scratch rows that map to it in sequence order and adds
//                      the sum once, so shared pages give the same bits on every run.
//   bwd_dq_kernel      query-major, shaped like the decode kernel (mma.m16n8k16, float32
//                      accumulators): a CTA owns up to 16 rows (the queries of a block times the G
//                      heads of one KV head), its four warps stream their own 16-key tiles (paged
//                      rows straight into smem by cp.async), and
//                        S^T = K Q^T, dP^T = V dO^T, dQ^T += K^T dS^T (dS^T to B fragments by
//                      movmatrix); the warps' dQ are summed in smem and written once.
#include "device_common.cuh"
#include "pa_internal.h"

namespace pa {

namespace {

constexpr int kBwdWarps = 4;
constexpr int kRowBlock = 16;             // rows per block (two n-tiles of 8)
constexpr int kDqStages = 3;

__device__ __forceinline__ int swz(int row, int chunk) { return chunk ^ (row & 7); }

constexpr float kLog2e = 1.4426950408889634f;

}  // namespace

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

// ---- dQ: a CTA per (block of up to 16 rows, KV head) -----------------------------------------
template <typename T, int D>
__global__ void __launch_bounds__(kBwdWarps * 32) bwd_dq_kernel(const BwdParams2 p) {
    constexpr int CH = D / 8, KK = D / 16, TT = 16;
    constexpr int TILE = TT * D, WARP_ELEMS = kDqStages * 2 * TILE;
    extern __shared__ __align__(128) uint8_t smem_raw[];
    T* smem = reinterpret_cast<T*>(smem_raw);

    const BwdRowUnit u = p.row_units[blockIdx.x];
    const int kvh = blockIdx.y;
    const SeqInfo si = p.seqs[u.seq];
    const int G = p.group;
    const int R = (u.j1 - u.j0) * G;  // live rows, <= 16
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int gq = lane >> 2, tq = lane & 3;
    const int64_t base_pos = (int64_t)si.L - si.n;
    auto qrow_of = [&](int r) { return (int64_t)(si.q_start + u.j0 + r / G) * p.hq + kvh * G + r % G; };

    // Q and dO rows as B fragments (column n = row gq of the n-tile)
    uint32_t qf[2][KK][2], of[2][KK][2];
    const T* qg = static_cast<const T*>(p.q);
    const T* og = static_cast<const T*>(p.dout);
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        const int r = nt * 8 + gq;
        const bool live = r < R;
        const int64_t qr = live ? qrow_of(r) : 0;
        const uint32_t* qs = reinterpret_cast<const uint32_t*>(qg + qr * D);
        const uint32_t* os = reinterpret_cast<const uint32_t*>(og + qr * D);
#pragma unroll
        for (int kk = 0; kk < KK; ++kk) {
            qf[nt][kk][0] = live ? qs[kk * 8 + tq] : 0u;
            qf[nt][kk][1] = live ? qs[kk * 8 + 4 + tq] : 0u;
            of[nt][kk][0] = live ? os[kk * 8 + tq] : 0u;
            of[nt][kk][1] = live ? os[kk * 8 + 4 + tq] : 0u;
        }
    }
    float lse2[2][2], dr[2][2];
    int64_t pos[2][2];
    bool livec[2][2];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            const int r = nt * 8 + 2 * tq + c;
            const bool live = r < R;
            const int64_t qr = live ? qrow_of(r) : 0;
            const float l = live ? p.lse[qr] : 0.f;
            livec[nt][c] = live && l != neg_inf();
            lse2[nt][c] = l * kLog2e;
            dr[nt][c] = livec[nt][c] ? p.drow[qr] : 0.f;
            pos[nt][c] = base_pos + u.j0 + (live ? r / G : 0);
        }
    // keys any of the rows can see: [lo, hi)
    const int64_t p_first = base_pos + u.j0, p_last = base_pos + u.j1 - 1;
    const int64_t lo = p.window > 0 ? max64(0, p_first - p.window + 1) : 0;
    const int64_t hi = p.causal ? min64(si.L, p_last + 1) : si.L;
    const int ntiles = hi > lo ? (int)((hi - lo + TT - 1) / TT) : 0;
    const int my_tiles = ntiles > warp ? (ntiles - warp + kBwdWarps - 1) / kBwdWarps : 0;

    float dq[KK][2][4];
#pragma unroll
    for (int dt = 0; dt < KK; ++dt)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) dq[dt][nt][0] = dq[dt][nt][1] = dq[dt][nt][2] = dq[dt][nt][3] = 0.f;

    T* wbuf = smem + (size_t)warp * WARP_ELEMS;
    const T* kc = static_cast<const T*>(p.k);
    const T* vc = static_cast<const T*>(p.v);
    const int32_t* bt = p.block_tables + (int64_t)u.seq * p.table_width;
    const int ps = p.page_size;
    const int64_t rstride = (int64_t)p.hkv * D;
    auto load_tile = [&](int it, int stage) {
        const int64_t tok0 = lo + (int64_t)(warp + it * kBwdWarps) * TT;
        int64_t off = -1;
        if (lane < TT) {
            const int64_t t = tok0 + lane;
            if (t < hi) off = ((int64_t)bt[t / ps] * ps + t % ps) * rstride + (int64_t)kvh * D;
        }
        T* dk = wbuf + stage * 2 * TILE;
        T* dv = dk + TILE;
#pragma unroll
        for (int c = lane; c < TT * CH; c += 32) {
            const int row = c / CH, ch = c % CH;
            const int64_t ro = __shfl_sync(0xffffffffu, off, row);
            const bool ok = ro >= 0;
            const int64_t src = ok ? ro + ch * 8 : 0;
            const int dst = row * D + swz(row, ch) * 8;
            cp_async_16(dk + dst, kc + src, ok);
            cp_async_16(dv + dst, vc + src, ok);
        }
    };
#pragma unroll
    for (int s = 0; s < kDqStages - 1; ++s) {
        if (s < my_tiles) load_tile(s, s);
        cp_async_commit();
    }
    for (int it = 0; it < my_tiles; ++it) {
        {
            const int nx = it + kDqStages - 1;
            if (nx < my_tiles) load_tile(nx, nx % kDqStages);
            cp_async_commit();
        }
        cp_async_wait<kDqStages - 1>();
        __syncwarp();
        const int stage = it % kDqStages;
        const T* sk = wbuf + stage * 2 * TILE;
        const T* sv = sk + TILE;
        const int64_t tok0 = lo + (int64_t)(warp + it * kBwdWarps) * TT;
        float s[2][4], dp[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) s[nt][e] = dp[nt][e] = 0.f;
#pragma unroll
        for (int kk = 0; kk < KK; ++kk) {
            uint32_t a[4];
            const int row = lane & 15;
            ldmatrix_x4(a, sk + row * D + swz(row, kk * 2 + (lane >> 4)) * 8);
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) mma16816<T>(s[nt], a, qf[nt][kk][0], qf[nt][kk][1]);
            ldmatrix_x4(a, sv + row * D + swz(row, kk * 2 + (lane >> 4)) * 8);
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) mma16816<T>(dp[nt], a, of[nt][kk][0], of[nt][kk][1]);
        }
        // dS^T -> B fragments of dS^T (keys as k, rows as n) through movmatrix
        uint32_t db[2][2];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            float dsv[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int c = e & 1;
                const int64_t t = tok0 + gq + 8 * (e >> 1);
                const bool vis = livec[nt][c] && t < hi && key_visible(t, pos[nt][c], p.causal, p.window);
                const float pr = vis ? fast_exp2(fmaf(s[nt][e], p.scale_log2, -lse2[nt][c])) : 0.f;
                dsv[e] = pr * (dp[nt][e] - dr[nt][c]);
            }
            db[nt][0] = movmatrix_trans(pack2<T>(dsv[0], dsv[1]));
            db[nt][1] = movmatrix_trans(pack2<T>(dsv[2], dsv[3]));
        }
        // dQ^T += K^T dS^T
#pragma unroll
        for (int dt = 0; dt < KK; ++dt) {
            uint32_t a[4];
            const int i = lane >> 3;
            const int row = (lane & 7) + 8 * (i >> 1);
            ldmatrix_x4_trans(a, sk + row * D + swz(row, dt * 2 + (i & 1)) * 8);
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) mma16816<T>(dq[dt][nt], a, db[nt][0], db[nt][1]);
        }
        __syncwarp();
    }
    cp_async_wait<0>();

    // ---- sum the warps' dQ and write it once ----
    __syncthreads();  // pipeline buffers are reused below
    float* eq = reinterpret_cast<float*>(smem_raw);  // [kBwdWarps][16][D]
#pragma unroll
    for (int dt = 0; dt < KK; ++dt)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int d = dt * 16 + gq + 8 * (e >> 1);
                const int r = nt * 8 + 2 * tq + (e & 1);
                eq[(warp * 16 + r) * D + d] = dq[dt][nt][e];
            }
    __syncthreads();
    for (int idx = threadIdx.x; idx < R * D; idx += kBwdWarps * 32) {
        const int r = idx / D, d = idx % D;
        float acc = 0.f;
#pragma unroll
        for (int w = 0; w < kBwdWarps; ++w) acc += eq[(w * 16 + r) * D + d];
        p.dq[qrow_of(r) * D + d] = acc * p.scale;
    }
}

// ---------------------------------------------------------------------------------------------
namespace {

template <typename T, int D>
cudaError_t bwd_launch_d(const BwdParams2& p, int num_key_units, int num_row_units, int64_t rows, int num_sums,
                         cudaStream_t st) {
    constexpr size_t dq_pipe = (size_t)kBwdWarps * kDqStages * 2 * 16 * D * sizeof(T);
    constexpr size_t dq_epi = (size_t)kBwdWarps * 16 * D * sizeof(float);
    constexpr size_t dq_smem = dq_pipe > dq_epi ? dq_pipe : dq_epi;
    static unsigned long long configured = 0;  // one bit per device ordinal
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 64 || !(configured >> dev & 1ull)) {
        e = cudaFuncSetAttribute(bwd_dq_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dq_smem);
        if (e != cudaSuccess) return e;
        if (dev < 64) configured |= 1ull << dev;
    }
    bwd_dot_kernel<T><<<(unsigned)((rows + 3) / 4), 128, 0, st>>>(static_cast<const T*>(p.out),
                                                                   static_cast<const T*>(p.dout), p.drow, rows, D);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (num_key_units > 0) {
        e = launch_backward_tc_dkdv(p, std::is_same<T, __nv_bfloat16>::value ? PA_BF16 : PA_F16, num_key_units,
                                    rows / p.hq, st);
        if (e != cudaSuccess) return e;
    }
    if (num_sums > 0)
        bwd_ordered_kernel<D><<<dim3((num_sums + 3) / 4, p.hkv), 128, 0, st>>>(p, num_sums, backward_tc_key_tile());
    if (num_row_units > 0)
        bwd_dq_kernel<T, D><<<dim3(num_row_units, p.hkv), kBwdWarps * 32, dq_smem, st>>>(p);
    return cudaGetLastError();
}

}  // namespace

bool backward_mma_supported(pa_dtype dt, int d, int dv, int group) {
    // dK/dV on tcgen05 walks 128-row blocks (128 / G queries x G heads); dQ takes <= 16 rows per CTA
    return (dt == PA_BF16 || dt == PA_F16) && d == dv && (d == 64 || d == 128) && group >= 1 &&
           group <= kRowBlock && 128 % group == 0;
}

int backward_key_tile() { return backward_tc_key_tile(); }
int backward_row_block() { return kRowBlock; }

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
