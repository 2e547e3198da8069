// Backward of paged GQA attention on the tensor cores (bf16 / fp16, D == Dv in {64, 128}, at most
// 16 query heads per KV head), deterministic and free of per-key atomics (boostr
// `standard_attention_bwd`; ruDNN's recompute-based backward, its "ordered" history pass in spirit:
// every key's gradient is summed by the one CTA that owns the key). With P recomputed from Q, K
// and the forward's lse (natural log), for each visible (row, key):
//     P = exp(scale q.k - lse),  dP = dO . v,  dS = P (dP - Drow),  Drow = dO . O
//     dV_k += P dO,   dK_k += scale dS q,   dQ_row += scale dS k
//
// Three kernels, all mma.m16n8k16 with float32 accumulators:
//   bwd_dot_kernel    Drow for every (query, head) row (a warp per row).
//   bwd_dkdv_kernel   key-major: a CTA owns 64 keys of one sequence and one KV head (a warp owns
//                     16 of them, their dK and dV rows in registers) and walks the 16-row blocks
//                     of (query, group head) rows that see those keys:
//                       S^T = K Q^T, dP^T = V dO^T   (keys as M, rows as N; K, V, Q, dO from smem)
//                       dV += P^T dO, dK += dS^T Q   (the S^T / dP^T accumulators are already the A
//                                                     fragments; dO and Q by ldmatrix.trans)
//                     and adds its 64 finished rows into the float32 gradient caches once (one add
//                     per element: the result does not depend on the order of CTAs unless two
//                     sequences share a page).
//   bwd_dq_kernel     query-major, shaped like the decode kernel: a CTA owns up to 16 rows (the
//                     queries of a block times the G heads of one KV head), its four warps stream
//                     their own 16-key tiles (paged rows straight into smem by cp.async), and
//                       S^T = K Q^T, dP^T = V dO^T, dQ^T += K^T dS^T (dS^T to B fragments by
//                     movmatrix); the warps' dQ are summed in smem and written once.
#include "device_common.cuh"
#include "pa_internal.h"

namespace pa {

namespace {

constexpr int kBwdWarps = 4;
constexpr int kKeyTile = 16 * kBwdWarps;  // keys per dK/dV CTA
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

// ---- dK, dV: a CTA per (64-key tile of a sequence, KV head) --------------------------------
template <typename T, int D>
__global__ void __launch_bounds__(kBwdWarps * 32) bwd_dkdv_kernel(const BwdParams2 p) {
    constexpr int CH = D / 8, KK = D / 16, NDT = D / 8;
    extern __shared__ __align__(128) uint8_t smem_raw[];
    T* sK = reinterpret_cast<T*>(smem_raw);
    T* sV = sK + kKeyTile * D;
    T* sQ = sV + kKeyTile * D;     // [2][16][D]
    T* sO = sQ + 2 * kRowBlock * D;  // [2][16][D] (the upstream gradient dO)
    int64_t* koff = reinterpret_cast<int64_t*>(sO + 2 * kRowBlock * D);  // [64] element offset of a key row

    const BwdKeyUnit u = p.key_units[blockIdx.x];
    const int kvh = blockIdx.y;
    const SeqInfo si = p.seqs[u.seq];
    const int G = p.group;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int gq = lane >> 2, tq = lane & 3;
    const int64_t k0 = u.k0;
    const int64_t kmax = min64(k0 + kKeyTile, si.L);  // keys [k0, kmax) exist
    const int64_t base_pos = (int64_t)si.L - si.n;    // position of query 0
    // queries that see at least one key of the tile: [j_lo, j_hi)
    int64_t j_lo = p.causal ? max64(0, k0 - base_pos) : 0;
    int64_t j_hi = p.window > 0 ? min64(si.n, kmax - 1 + p.window - base_pos) : si.n;
    if (j_hi <= j_lo || kmax <= k0) return;  // nothing to add
    const int64_t R_lo = j_lo * G, R_hi = j_hi * G;
    const int rb0 = (int)(R_lo / kRowBlock), rb1 = (int)((R_hi + kRowBlock - 1) / kRowBlock);

    const int32_t* bt = p.block_tables + (int64_t)u.seq * p.table_width;
    const int ps = p.page_size;
    const int64_t rstride = (int64_t)p.hkv * D;
    if (tid < kKeyTile) {
        const int64_t t = k0 + tid;
        koff[tid] = t < kmax ? ((int64_t)bt[t / ps] * ps + t % ps) * rstride + (int64_t)kvh * D : -1;
    }
    __syncthreads();
    const T* kc = static_cast<const T*>(p.k);
    const T* vc = static_cast<const T*>(p.v);
    for (int c = tid; c < kKeyTile * CH; c += kBwdWarps * 32) {
        const int row = c / CH, ch = c % CH;
        const int64_t ro = koff[row];
        const bool ok = ro >= 0;
        const int64_t src = ok ? ro + ch * 8 : 0;
        const int dst = row * D + swz(row, ch) * 8;
        cp_async_16(sK + dst, kc + src, ok);
        cp_async_16(sV + dst, vc + src, ok);
    }
    const T* qg = static_cast<const T*>(p.q);
    const T* og = static_cast<const T*>(p.dout);
    // rows of a sequence (queries x G) stay below 2^31 (the host checks), so row -> (query, head)
    // is a 32-bit division
    const uint32_t Gu = (uint32_t)G;
    auto qrow_of = [&](int64_t R) {
        const uint32_t r = (uint32_t)R, j = r / Gu;
        return (int64_t)(si.q_start + (int64_t)j) * p.hq + kvh * G + (int)(r - j * Gu);
    };
    auto load_rows = [&](int rb, int st) {
        for (int c = tid; c < 2 * kRowBlock * CH; c += kBwdWarps * 32) {
            const int which = c / (kRowBlock * CH), rc = c % (kRowBlock * CH);
            const int i = rc / CH, ch = rc % CH;
            const int64_t R = (int64_t)rb * kRowBlock + i;
            const bool ok = R >= R_lo && R < R_hi;
            const int64_t src = ok ? qrow_of(R) * D + ch * 8 : 0;
            T* dst = (which ? sO : sQ) + st * kRowBlock * D + i * D + swz(i, ch) * 8;
            cp_async_16(dst, (which ? og : qg) + src, ok);
        }
    };
    load_rows(rb0, 0);
    cp_async_commit();

    float dk[NDT][4], dv[NDT][4];
#pragma unroll
    for (int n = 0; n < NDT; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) dk[n][e] = dv[n][e] = 0.f;
    const int kw = warp * 16;  // this warp's first key row in the tile

    // lse and Drow of this thread's four rows (two per n-tile) of a block; the next block's are
    // loaded while the current one computes
    float lse_n[2][2], dr_n[2][2];
    auto row_stats = [&](int rb) {
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                const int64_t R = (int64_t)rb * kRowBlock + nt * 8 + 2 * tq + c;
                const bool in = R >= R_lo && R < R_hi;
                const int64_t qr = in ? qrow_of(R) : 0;
                lse_n[nt][c] = in ? p.lse[qr] : neg_inf();
                dr_n[nt][c] = in ? p.drow[qr] : 0.f;
            }
    };
    row_stats(rb0);
    for (int rb = rb0; rb < rb1; ++rb) {
        const int st = (rb - rb0) & 1;
        if (rb + 1 < rb1) load_rows(rb + 1, st ^ 1);
        cp_async_commit();
        // this block's rows: lse in base 2, Drow, position, liveness (a row without keys has lse -inf)
        float lse2[2][2], dr[2][2];
        int64_t pos[2][2];
        bool live[2][2];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                const int64_t R = (int64_t)rb * kRowBlock + nt * 8 + 2 * tq + c;
                live[nt][c] = lse_n[nt][c] != neg_inf();
                lse2[nt][c] = live[nt][c] ? lse_n[nt][c] * kLog2e : 0.f;
                dr[nt][c] = dr_n[nt][c];
                pos[nt][c] = base_pos + (live[nt][c] ? (int64_t)((uint32_t)R / Gu) : 0);
            }
        // every row of the block live and seeing every key of the tile: no per-element mask
        const int64_t r_first = (int64_t)rb * kRowBlock, r_last = r_first + kRowBlock - 1;
        const int64_t pmin = base_pos + (int64_t)((uint32_t)r_first / Gu);
        const int64_t pmax = base_pos + (int64_t)((uint32_t)r_last / Gu);
        const bool full = kmax == k0 + kKeyTile && r_first >= R_lo && r_last < R_hi && (!p.causal || kmax - 1 <= pmin) &&
                          (p.window == 0 || k0 + p.window > pmax) &&
                          __all_sync(0xffffffffu, live[0][0] && live[0][1] && live[1][0] && live[1][1]);
        if (rb + 1 < rb1) row_stats(rb + 1);
        cp_async_wait<1>();
        __syncthreads();
        const T* q_s = sQ + st * kRowBlock * D;
        const T* o_s = sO + st * kRowBlock * D;
        // ---- S^T = K Q^T and dP^T = V dO^T (16 keys x 16 rows) ----
        float s[2][4], dp[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) s[nt][e] = dp[nt][e] = 0.f;
#pragma unroll
        for (int kk = 0; kk < KK; ++kk) {
            uint32_t a[4], b[4];
            const int arow = kw + (lane & 15);
            const int i = lane >> 3;
            const int brow = (lane & 7) + 8 * (i >> 1);
            ldmatrix_x4(a, sK + arow * D + swz(arow, kk * 2 + (lane >> 4)) * 8);
            ldmatrix_x4(b, q_s + brow * D + swz(brow, kk * 2 + (i & 1)) * 8);
            mma16816<T>(s[0], a, b[0], b[1]);
            mma16816<T>(s[1], a, b[2], b[3]);
            ldmatrix_x4(a, sV + arow * D + swz(arow, kk * 2 + (lane >> 4)) * 8);
            ldmatrix_x4(b, o_s + brow * D + swz(brow, kk * 2 + (i & 1)) * 8);
            mma16816<T>(dp[0], a, b[0], b[1]);
            mma16816<T>(dp[1], a, b[2], b[3]);
        }
        // ---- P^T and dS^T, packed as the A fragments of the two products below ----
        uint32_t pa[4], da[4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            float pv[4], dsv[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int c = e & 1;
                const int64_t t = k0 + kw + gq + 8 * (e >> 1);
                const bool vis =
                    full || (live[nt][c] && t < kmax && key_visible(t, pos[nt][c], p.causal, p.window));
                const float pr = vis ? fast_exp2(fmaf(s[nt][e], p.scale_log2, -lse2[nt][c])) : 0.f;
                pv[e] = pr;
                dsv[e] = pr * (dp[nt][e] - dr[nt][c]);
            }
            pa[nt * 2 + 0] = pack2<T>(pv[0], pv[1]);
            pa[nt * 2 + 1] = pack2<T>(pv[2], pv[3]);
            da[nt * 2 + 0] = pack2<T>(dsv[0], dsv[1]);
            da[nt * 2 + 1] = pack2<T>(dsv[2], dsv[3]);
        }
        // A fragment order: (keys 0-7, rows 0-7), (keys 8-15, rows 0-7), (keys 0-7, rows 8-15), (keys 8-15, rows 8-15)
        const uint32_t pA[4] = {pa[0], pa[1], pa[2], pa[3]};
        const uint32_t dA[4] = {da[0], da[1], da[2], da[3]};
        // ---- dV += P^T dO and dK += dS^T Q (k = the 16 rows, n = 8 columns of D) ----
#pragma unroll
        for (int dp2 = 0; dp2 < D / 16; ++dp2) {
            uint32_t b[4];
            const int i = lane >> 3;
            const int row = (lane & 7) + 8 * (i & 1);
            ldmatrix_x4_trans(b, o_s + row * D + swz(row, dp2 * 2 + (i >> 1)) * 8);
            mma16816<T>(dv[2 * dp2], pA, b[0], b[1]);
            mma16816<T>(dv[2 * dp2 + 1], pA, b[2], b[3]);
            ldmatrix_x4_trans(b, q_s + row * D + swz(row, dp2 * 2 + (i >> 1)) * 8);
            mma16816<T>(dk[2 * dp2], dA, b[0], b[1]);
            mma16816<T>(dk[2 * dp2 + 1], dA, b[2], b[3]);
        }
        __syncthreads();  // the stage is loaded again two blocks on
    }
    cp_async_wait<0>();

    // ---- add the tile's rows into the gradient caches (one add per element) ----
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int r = kw + gq + 8 * h;
        const int64_t ro = koff[r];
        if (ro < 0) continue;
        float* dkr = p.dk + ro;
        float* dvr = p.dv + ro;
#pragma unroll
        for (int n = 0; n < NDT; ++n) {
            const int d = n * 8 + 2 * tq;
            atomicAdd(dkr + d, dk[n][2 * h] * p.scale);
            atomicAdd(dkr + d + 1, dk[n][2 * h + 1] * p.scale);
            atomicAdd(dvr + d, dv[n][2 * h]);
            atomicAdd(dvr + d + 1, dv[n][2 * h + 1]);
        }
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
cudaError_t bwd_launch_d(const BwdParams2& p, int num_key_units, int num_row_units, int64_t rows, cudaStream_t st) {
    constexpr size_t kv_smem = (size_t)(2 * kKeyTile + 4 * kRowBlock) * D * sizeof(T) + kKeyTile * sizeof(int64_t);
    constexpr size_t dq_pipe = (size_t)kBwdWarps * kDqStages * 2 * 16 * D * sizeof(T);
    constexpr size_t dq_epi = (size_t)kBwdWarps * 16 * D * sizeof(float);
    constexpr size_t dq_smem = dq_pipe > dq_epi ? dq_pipe : dq_epi;
    static unsigned long long configured = 0;  // one bit per device ordinal
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 64 || !(configured >> dev & 1ull)) {
        e = cudaFuncSetAttribute(bwd_dkdv_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kv_smem);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(bwd_dq_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dq_smem);
        if (e != cudaSuccess) return e;
        if (dev < 64) configured |= 1ull << dev;
    }
    bwd_dot_kernel<T><<<(unsigned)((rows + 3) / 4), 128, 0, st>>>(static_cast<const T*>(p.out),
                                                                   static_cast<const T*>(p.dout), p.drow, rows, D);
    if (num_key_units > 0)
        bwd_dkdv_kernel<T, D><<<dim3(num_key_units, p.hkv), kBwdWarps * 32, kv_smem, st>>>(p);
    if (num_row_units > 0)
        bwd_dq_kernel<T, D><<<dim3(num_row_units, p.hkv), kBwdWarps * 32, dq_smem, st>>>(p);
    return cudaGetLastError();
}

}  // namespace

bool backward_mma_supported(pa_dtype dt, int d, int dv, int group) {
    return (dt == PA_BF16 || dt == PA_F16) && d == dv && (d == 64 || d == 128) && group >= 1 && group <= kRowBlock;
}

int backward_key_tile() { return kKeyTile; }
int backward_row_block() { return kRowBlock; }

cudaError_t launch_backward_mma(const BwdParams2& p, pa_dtype dt, int num_key_units, int num_row_units, int64_t rows,
                                cudaStream_t st) {
    if (rows == 0) return cudaSuccess;
    if (dt == PA_BF16)
        return p.d == 64 ? bwd_launch_d<__nv_bfloat16, 64>(p, num_key_units, num_row_units, rows, st)
                         : bwd_launch_d<__nv_bfloat16, 128>(p, num_key_units, num_row_units, rows, st);
    return p.d == 64 ? bwd_launch_d<__half, 64>(p, num_key_units, num_row_units, rows, st)
                     : bwd_launch_d<__half, 128>(p, num_key_units, num_row_units, rows, st);
}

}  // namespace pa
