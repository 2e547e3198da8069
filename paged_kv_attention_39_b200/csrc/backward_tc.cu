// dK, dV and dQ of paged GQA attention on the 5th-generation tensor cores (tcgen05 + TMEM + TMA),
// bf16 / fp16, head_dim == v_head_dim in {64, 128}, G dividing 128 (boostr
// `standard_attention_bwd`; ruDNN's recompute-based backward). With P recomputed from Q, K and the
// forward's lse (natural log), for every visible (row, key):
//     P = exp(scale q.k - lse),  dP = dO . v,  dS = P (dP - Drow),  Drow = dO . O
//     dV_k += P dO,   dK_k += scale dS q
//
// Key-major: a CTA owns 128 keys of one sequence and one KV head and walks the blocks of 128 rows
// (128 / G queries x the G heads of the KV head, the prefill kernels' tile) that see those keys:
//   S^T  = K Q^T       (M = 128 keys, N = 128 rows, K = D)   -> TMEM columns [0, 128)
//   dP^T = V dO^T                                            -> TMEM columns [128, 256)
//   P^T, dS^T in float32 by the four compute warps (thread = key), rounded to 16 bits and written
//   over the first 64 columns of their own buffers
//   dV  += P^T dO      (A = P^T from TMEM, B = dO, MN-major)  -> TMEM columns [256, 256 + D)
//   dK  += dS^T Q      (A = dS^T from TMEM, B = Q)            -> TMEM columns [256 + D, 256 + 2D)
// and at the end adds its finished rows once into the float32 gradient caches (the only writer of
// those rows), or, for a tile the host marked ordered (it touches a shared page), writes them to
// the scratch the ordered pass sums. dQ comes from the query-major kernel at the end of this file.
//
//   warps 0..7  compute: row statistics from shared memory, masks, P and dS, the epilogue (two
//               warps per 32 keys, each taking half of the block's rows and of the dK/dV columns)
//   warp 8      loads: the K and V rows of the tile once (TMA, one box per page), then per row
//               block the Q and dO rows (TMA, two stages) and the block's lse, Drow and visible
//               key ranges (into shared memory)
//   warp 9      TMEM owner and MMA issuer (one thread)
//
// Every wait on an mbarrier is bounded (Watchdog): a stalled pipeline sets the plan's error word and
// the CTA leaves through its normal exit, freeing TMEM.
#include <cudaTypedefs.h>

#include "sm100.cuh"

namespace pa {

using namespace sm100;

namespace {

constexpr int KT = 128;  // keys per CTA
constexpr int RB = 128;  // rows per block
constexpr int QST = 2;   // Q / dO stages
// warps 0..7 compute (two per TMEM lane quadrant: warp w reaches lanes 32 (w % 4) .. and takes
// half w / 4 of the block's columns), warp 8 loads, warp 9 owns TMEM and issues the MMAs
constexpr int kComputeWarpsB = 8, kLoadWarp = 8, kMmaWarp = 9, kThreadsB = 10 * 32;
constexpr uint32_t kTmemColsB = 512;
constexpr uint64_t kWaitLimitNsB = 2000000000ull;
constexpr float kLog2eB = 1.4426950408889634f;

template <int D>
struct BtcCfg {
    static constexpr int KH = D / 64;       // 128-byte halves of a row
    static constexpr int HALF = 128 * 128;  // bytes of one half of a 128-row tile
    static constexpr int K = 0;
    static constexpr int V = K + KH * HALF;
    static constexpr int Q = V + KH * HALF;          // stage s: Q at Q + s * 2 * KH * HALF, dO after it
    static constexpr int ROWS = Q + QST * 2 * KH * HALF;  // stage s: lse2, drow, lo, hi (128 each) + 2 ints
    static constexpr int ROWS_STAGE = 4 * RB * 4 + 16;
    static constexpr int BAR = ROWS + QST * ROWS_STAGE;
    static constexpr int BYTES = BAR + 256;
    static constexpr int ALLOC = BYTES + 1024;
    static_assert(ALLOC <= 232448, "shared memory of one CTA");
    static_assert(2 * (D / 32) * 128 * 128 <= QST * 2 * KH * HALF, "dK / dV staging fits over the Q / dO stages");
    static constexpr int T_ST = 0, T_DPT = 128, T_DV = 256, T_DK = 256 + D;
    static constexpr int B_KV = 0, B_QFULL = 1, B_QEMPTY = B_QFULL + QST, B_SFULL = B_QEMPTY + QST,
                         B_PFULL = B_SFULL + 1, B_DONE = B_PFULL + 1, B_COUNT = B_DONE + 1;
};

__device__ __forceinline__ int btc_swz(int row, int chunk) { return chunk ^ (row & 7); }

// TMEM column of row `row` of a block's packed P^T / dS^T (two 16-bit rows per column; the second
// half of the rows sits over the third quarter of the buffer)
__host__ __device__ constexpr int packed_col(int row) { return row / 2 + (row >= RB / 2 ? RB / 4 : 0); }

}  // namespace

// P^T and dS^T of one key (thread = TMEM lane) against rows [32 c0, 32 c1) of a block, 16-bit,
// packed two rows per column over columns of the S^T and dP^T buffers that this warp has read
// (rows [0, 64) -> columns [0, 32), rows [64, 128) -> columns [64, 96): the two warps of a lane
// quadrant each read and write only their own half of a buffer). The rows' statistics come from shared
// memory four at a time (one 16-byte load per statistic for four rows); MASKED adds each row's
// visible key range [lo, hi) (a row without keys has lo = hi = 0).
template <typename T, bool MASKED>
__device__ __forceinline__ void btc_probs(uint32_t t_lane, const float* lse2, const float* drow, const int* lo,
                                          const int* hi, int64_t t, float scale_log2, int c0, int c1) {
#pragma unroll 1
    for (int c = c0; c < c1; ++c) {
        uint32_t sv[32], dv[32];
        tmem_ld32(t_lane + BtcCfg<64>::T_ST + c * 32, sv);
        tmem_ld32(t_lane + BtcCfg<64>::T_DPT + c * 32, dv);
        tmem_ld_wait(sv);
        tmem_regs_ready(dv);
        uint32_t pk[16], dk[16];
#pragma unroll
        for (int q = 0; q < 8; ++q) {  // rows c*32 + 4q .. + 3
            const float4 l4 = *reinterpret_cast<const float4*>(lse2 + c * 32 + 4 * q);
            const float4 d4 = *reinterpret_cast<const float4*>(drow + c * 32 + 4 * q);
            const float lv[4] = {l4.x, l4.y, l4.z, l4.w}, dr[4] = {d4.x, d4.y, d4.z, d4.w};
            bool vis[4] = {true, true, true, true};
            if (MASKED) {
                const int4 a4 = *reinterpret_cast<const int4*>(lo + c * 32 + 4 * q);
                const int4 b4 = *reinterpret_cast<const int4*>(hi + c * 32 + 4 * q);
                vis[0] = t >= a4.x && t < b4.x;
                vis[1] = t >= a4.y && t < b4.y;
                vis[2] = t >= a4.z && t < b4.z;
                vis[3] = t >= a4.w && t < b4.w;
            }
            float pr[4], ds[4];
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                const float pv = fast_exp2(fmaf(__uint_as_float(sv[4 * q + x]), scale_log2, -lv[x]));
                pr[x] = vis[x] ? pv : 0.f;
                ds[x] = vis[x] ? pv * (__uint_as_float(dv[4 * q + x]) - dr[x]) : 0.f;
            }
            pk[2 * q] = pack2<T>(pr[0], pr[1]);
            pk[2 * q + 1] = pack2<T>(pr[2], pr[3]);
            dk[2 * q] = pack2<T>(ds[0], ds[1]);
            dk[2 * q + 1] = pack2<T>(ds[2], ds[3]);
        }
        // 32 row-columns -> 16 TMEM columns, over columns already read
        const int pc = packed_col(c * 32);
        tmem_st16(t_lane + BtcCfg<64>::T_ST + pc, pk);
        tmem_st16(t_lane + BtcCfg<64>::T_DPT + pc, dk);
    }
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreadsB, 1)
    bwd_tc_dkdv_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmo,
                       const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                       const __grid_constant__ CUtensorMap tmdk, const __grid_constant__ CUtensorMap tmdv,
                       const BwdParams2 p) {
    using L_ = BtcCfg<D>;
    constexpr int KH = L_::KH;
    constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
    constexpr uint32_t IDESC_S = idesc_f16(KT, RB, kBf16, false, false);
    constexpr uint32_t IDESC_G = idesc_f16(KT, D, kBf16, false, true);

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L_::BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + L_::B_COUNT);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    const Watchdog wd{abort_flag, p.err, kWaitLimitNsB};

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const BwdKeyUnit u = p.key_units[blockIdx.x];
    const int kvh = blockIdx.y;
    const SeqInfo si = p.seqs[u.seq];
    const int G = p.group, qpt = RB / G;
    const int64_t k0 = u.k0;
    const int64_t kmax = min64(k0 + KT, si.L);       // keys [k0, kmax) exist
    const int64_t base_pos = (int64_t)si.L - si.n;   // position of query 0
    // queries that see at least one key of the tile: [j_lo, j_hi), in blocks of qpt
    const int64_t j_lo = p.causal ? max64(0, k0 - base_pos) : 0;
    const int64_t j_hi = p.window > 0 ? min64(si.n, kmax - 1 + p.window - base_pos) : si.n;
    const int rb0 = (int)(j_lo / qpt);
    const int nblk = j_hi > j_lo ? (int)((j_hi + qpt - 1) / qpt) - rb0 : 0;

    if (tid == 0) {
        for (int i = 0; i < L_::B_COUNT; ++i) {
            uint32_t cnt = 1;
            if (i == L_::B_PFULL) cnt = kComputeWarpsB * 32;
            if (i >= L_::B_QFULL && i < L_::B_QFULL + QST) cnt = 2;  // tile bytes + row statistics
            mbar_init(&bars[i], cnt);
        }
        *abort_flag = 0;
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(tmem_slot, kTmemColsB);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t s_base = smem_u32(smem);

    if (warp == kLoadWarp) {
        // ===================== loads =====================
        if (lane == 0) {
            tma_prefetch(&tmq);
            tma_prefetch(&tmo);
        }
        // the row block's Q and dO rows (TMA) and its row statistics (plain loads) into stage s
        auto load_block = [&](int i, int s) {
            const int j0 = (rb0 + i) * qpt;
            // the tiles first: their landing is what the block waits for; the row statistics are
            // gathered while they are in flight and reported by a second arrival
            if (lane == 0) {
                mbar_arrive_expect_tx(&bars[L_::B_QFULL + s], 2 * KH * L_::HALF);
                uint8_t* qs = smem + L_::Q + s * 2 * KH * L_::HALF;
                for (int h = 0; h < KH; ++h) {
                    tma_load_3d(qs + h * L_::HALF, &tmq, &bars[L_::B_QFULL + s], h * 64, kvh * G, si.q_start + j0);
                    tma_load_3d(qs + (KH + h) * L_::HALF, &tmo, &bars[L_::B_QFULL + s], h * 64, kvh * G,
                                si.q_start + j0);
                }
            }
            uint8_t* rows = smem + L_::ROWS + s * L_::ROWS_STAGE;
            float* lse2 = reinterpret_cast<float*>(rows);
            float* drow = lse2 + RB;
            int* lo = reinterpret_cast<int*>(drow + RB);
            int* hi = lo + RB;
            int lo_max = 0, hi_min = INT32_MAX;
            for (int r = lane; r < RB; r += 32) {
                const int j = j0 + r / G;
                const bool live = j < si.n;
                const int64_t qr = (int64_t)(si.q_start + (live ? j : 0)) * p.hq + kvh * G + r % G;
                const float l = live ? p.lse[qr] : neg_inf();
                const bool has = live && l != neg_inf();
                const int64_t pos = base_pos + j;
                const int64_t a = p.window > 0 ? max64(0, pos - p.window + 1) : 0;
                const int64_t b = p.causal ? min64(si.L, pos + 1) : si.L;
                lse2[r] = has ? l * kLog2eB : 0.f;
                drow[r] = has ? p.drow[qr] : 0.f;
                lo[r] = has ? (int)a : 0;
                hi[r] = has ? (int)b : 0;
                lo_max = max(lo_max, lo[r]);
                hi_min = min(hi_min, hi[r]);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                lo_max = max(lo_max, __shfl_xor_sync(0xffffffffu, lo_max, o));
                hi_min = min(hi_min, __shfl_xor_sync(0xffffffffu, hi_min, o));
            }
            if (lane == 0) {
                hi[RB] = lo_max;  // every row sees [lo_max, hi_min)
                hi[RB + 1] = hi_min;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[L_::B_QFULL + s]);  // the statistics are written
            __syncwarp();
        };
        // the tile's K and V rows: one TMA box per page (and 64-column half), landing 128-byte
        // swizzled at rows b * kbox .. of the tile. Boxes past the sequence's last page are not
        // loaded: those keys are masked (P and dS select zero), and their dK / dV rows are zero.
        const int ps = p.page_size, kbox = ps < KT ? ps : KT;
        const int nbox = (int)((kmax - k0 + kbox - 1) / kbox);  // at most KT / 16 boxes
        {
            const int32_t* bt = p.block_tables + (int64_t)u.seq * p.table_width;
            int my_row = 0;
            if (lane < nbox) {
                const int64_t key = k0 + (int64_t)lane * kbox;
                my_row = bt[key / ps] * ps + (int)(key % ps);
            }
            if (lane == 0) {
                tma_prefetch(&tmk);
                tma_prefetch(&tmv);
                mbar_arrive_expect_tx(&bars[L_::B_KV], (uint32_t)(nbox * kbox * 128 * KH * 2));
            }
            for (int b = 0; b < nbox; ++b) {
                const int row = __shfl_sync(0xffffffffu, my_row, b);
                if (lane == 0)
                    for (int h = 0; h < KH; ++h) {
                        tma_load_3d(smem + L_::K + h * L_::HALF + b * kbox * 128, &tmk, &bars[L_::B_KV], h * 64, kvh, row);
                        tma_load_3d(smem + L_::V + h * L_::HALF + b * kbox * 128, &tmv, &bars[L_::B_KV], h * 64, kvh, row);
                    }
            }
            __syncwarp();
        }
        bool ok = true;
        for (int i = 0; i < nblk && i < QST; ++i) load_block(i, i);
        for (int i = QST; ok && i < nblk; ++i) {
            const int s = i % QST;
            ok = __all_sync(0xffffffffu, mbar_wait(&bars[L_::B_QEMPTY + s], ((i / QST) - 1) & 1, wd, 21));
            if (ok) load_block(i, s);
        }
        if (lane == 0 && *abort_flag) {
            // leave no copy in flight into this CTA's shared memory (bounded, ignoring the flag)
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(&bars[L_::B_KV], 0) && globaltimer_ns() - t0 < kWaitLimitNsB) {}
            for (int i = max(0, nblk - QST); i < nblk; ++i)
                while (!mbar_try_wait(&bars[L_::B_QFULL + i % QST], (i / QST) & 1) && globaltimer_ns() - t0 < kWaitLimitNsB) {}
        }
    } else if (warp == kMmaWarp) {
        // ===================== MMA issuer =====================
        const uint64_t dK = sdesc_sw128(s_base + L_::K, 16, 1024);
        const uint64_t dV = sdesc_sw128(s_base + L_::V, 16, 1024);
        bool ok = nblk == 0 || __all_sync(0xffffffffu, mbar_wait(&bars[L_::B_KV], 0, wd, 22));
        for (int i = 0; ok && i < nblk; ++i) {
            const int s = i % QST;
            // S^T and dP^T of this block overwrite P^T / dS^T of the previous one: its products are done
            if (i > 0) ok = __all_sync(0xffffffffu, mbar_wait(&bars[L_::B_DONE], (i - 1) & 1, wd, 23));
            if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bars[L_::B_QFULL + s], (i / QST) & 1, wd, 24));
            if (!ok) break;
            tc_fence_after();
            const uint32_t qs = s_base + L_::Q + s * 2 * KH * L_::HALF;
            const uint32_t os = qs + KH * L_::HALF;
            if (lane == 0) {
                const uint64_t dQk = sdesc_sw128(qs, 16, 1024), dOk = sdesc_sw128(os, 16, 1024);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * L_::HALF + (kk & 3) * 32;
                    mma_f16_ss(tmem + L_::T_ST, desc_add(dK, off), desc_add(dQk, off), IDESC_S, kk > 0);
                    mma_f16_ss(tmem + L_::T_DPT, desc_add(dV, off), desc_add(dOk, off), IDESC_S, kk > 0);
                }
                mma_commit(&bars[L_::B_SFULL]);
            }
            __syncwarp();
            ok = __all_sync(0xffffffffu, mbar_wait(&bars[L_::B_PFULL], i & 1, wd, 25));
            if (!ok) break;
            tc_fence_after();
            if (lane == 0) {
                // rows are the contraction: 16 rows = 8 TMEM columns of P^T / dS^T, 2 KB of dO / Q
                const uint64_t dOn = sdesc_sw128(os, L_::HALF, 1024), dQn = sdesc_sw128(qs, L_::HALF, 1024);
#pragma unroll
                for (int kk = 0; kk < RB / 16; ++kk) {
                    const uint32_t acc = (i > 0 || kk > 0) ? 1u : 0u;
                    mma_f16_ts(tmem + L_::T_DV, tmem + L_::T_ST + packed_col(kk * 16), desc_add(dOn, kk * 16 * 128),
                               IDESC_G, acc);
                    mma_f16_ts(tmem + L_::T_DK, tmem + L_::T_DPT + packed_col(kk * 16), desc_add(dQn, kk * 16 * 128),
                               IDESC_G, acc);
                }
                mma_commit(&bars[L_::B_DONE]);
                mma_commit(&bars[L_::B_QEMPTY + s]);
            }
            __syncwarp();
        }
    } else {
        // ===================== compute: thread = key =====================
        const int hf = warp >> 2;        // this warp's half of the block's rows / of the dK, dV columns
        const int r0 = (warp & 3) * 32;  // this warp's TMEM lanes (keys k0 + r0 ..)
        const uint32_t lane_off = (uint32_t)r0 << 16;
        const int64_t t = k0 + r0 + lane;  // this thread's key
        const int64_t tw0 = k0 + r0, tw1 = k0 + r0 + 31;
        bool ok = true;
        for (int i = 0; i < nblk; ++i) {
            const int s = i % QST;
            ok = __all_sync(0xffffffffu, mbar_wait(&bars[L_::B_QFULL + s], (i / QST) & 1, wd, 26)) && ok;
            ok = __all_sync(0xffffffffu, mbar_wait(&bars[L_::B_SFULL], i & 1, wd, 27)) && ok;
            tc_fence_after();
            const uint8_t* rows = smem + L_::ROWS + s * L_::ROWS_STAGE;
            const float* lse2 = reinterpret_cast<const float*>(rows);
            const float* drow = lse2 + RB;
            const int* lo = reinterpret_cast<const int*>(drow + RB);
            const int* hi = lo + RB;
            // every key of the warp seen by every row of the block: no per-element mask (keys past the
            // sequence's end are outside every row's range, so they always take the masked path)
            const bool full = tw1 < kmax && tw0 >= hi[RB] && tw1 < hi[RB + 1];
            if (__all_sync(0xffffffffu, full))
                btc_probs<T, false>(tmem + lane_off, lse2, drow, lo, hi, t, p.scale_log2, hf * RB / 64, (hf + 1) * RB / 64);
            else
                btc_probs<T, true>(tmem + lane_off, lse2, drow, lo, hi, t, p.scale_log2, hf * RB / 64, (hf + 1) * RB / 64);
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(&bars[L_::B_PFULL]);
        }
        // ---- epilogue: the tile's finished dK / dV rows ----
        if (nblk > 0 && ok) ok = __all_sync(0xffffffffu, mbar_wait(&bars[L_::B_DONE], (nblk - 1) & 1, wd, 28));
        ok = __all_sync(0xffffffffu, ok);
        tc_fence_after();
        if (ok && nblk > 0 && u.ord >= 0) {
            // a tile touching a shared page: its rows go to scratch, summed later by the ordered pass
            const int64_t srow = ((int64_t)u.ord * p.hkv + kvh) * KT + r0 + lane;
            float* dk_row = p.scratch_k + srow * D;
            float* dv_row = p.scratch_v + srow * D;
#pragma unroll 1
            for (int c = hf * (D / 64); c < (hf + 1) * (D / 64); ++c) {
                uint32_t a[32], b[32];
                tmem_ld32(tmem + L_::T_DV + lane_off + c * 32, a);
                tmem_ld32(tmem + L_::T_DK + lane_off + c * 32, b);
                tmem_ld_wait(a);
                tmem_regs_ready(b);
                float4* kd = reinterpret_cast<float4*>(dk_row + c * 32);
                float4* vd = reinterpret_cast<float4*>(dv_row + c * 32);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    kd[e] = make_float4(__uint_as_float(b[4 * e]) * p.scale, __uint_as_float(b[4 * e + 1]) * p.scale,
                                        __uint_as_float(b[4 * e + 2]) * p.scale, __uint_as_float(b[4 * e + 3]) * p.scale);
                    vd[e] = make_float4(__uint_as_float(a[4 * e]), __uint_as_float(a[4 * e + 1]),
                                        __uint_as_float(a[4 * e + 2]), __uint_as_float(a[4 * e + 3]));
                }
            }
        } else if (ok && nblk > 0) {
            // This CTA is the only writer of its rows: stage them in shared memory (over the Q / dO
            // stages, idle now) as 128-byte swizzled 32-column blocks of the 128 rows, then add them
            // onto the caller's cache with TMA reduce-adds, one box per page and column block (one
            // add per element; keys past the sequence's end add zeros to their own page's rows).
            // Each warp takes its 32 rows and its half of the column blocks.
            constexpr int CB = 128 * 128;  // one 32-column block of the 128 rows, float32
            uint8_t* stg_v = smem + L_::Q;
            uint8_t* stg_k = stg_v + (D / 32) * CB;
            const int r = r0 + lane;
#pragma unroll 1
            for (int c = hf * (D / 64); c < (hf + 1) * (D / 64); ++c) {
                uint32_t a[32], b[32];
                tmem_ld32(tmem + L_::T_DV + lane_off + c * 32, a);
                tmem_ld32(tmem + L_::T_DK + lane_off + c * 32, b);
                tmem_ld_wait(a);
                tmem_regs_ready(b);
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    const int off = c * CB + r * 128 + (btc_swz(r, ch) << 4);
                    *reinterpret_cast<float4*>(stg_v + off) =
                        make_float4(__uint_as_float(a[4 * ch]), __uint_as_float(a[4 * ch + 1]),
                                    __uint_as_float(a[4 * ch + 2]), __uint_as_float(a[4 * ch + 3]));
                    *reinterpret_cast<float4*>(stg_k + off) =
                        make_float4(__uint_as_float(b[4 * ch]) * p.scale, __uint_as_float(b[4 * ch + 1]) * p.scale,
                                    __uint_as_float(b[4 * ch + 2]) * p.scale, __uint_as_float(b[4 * ch + 3]) * p.scale);
                }
            }
            fence_proxy_async_smem();  // the staged rows are read by the TMA engine
            __syncwarp();
            if (lane == 0) {
                const int ps = p.page_size, rbox = ps < 32 ? ps : 32;
                const int32_t* bt = p.block_tables + (int64_t)u.seq * p.table_width;
                for (int b0 = 0; b0 < 32; b0 += rbox) {  // this warp's 32 rows, one box per page
                    const int64_t key = k0 + r0 + b0;
                    if (key >= kmax) break;
                    const int row = bt[key / ps] * ps + (int)(key % ps);
                    for (int c = hf * (D / 64); c < (hf + 1) * (D / 64); ++c) {
                        tma_reduce_add_3d(&tmdv, stg_v + c * CB + (r0 + b0) * 128, c * 32, kvh, row);
                        tma_reduce_add_3d(&tmdk, stg_k + c * CB + (r0 + b0) * 128, c * 32, kvh, row);
                    }
                }
                bulk_commit_group();
                bulk_wait_all();
            }
            __syncwarp();
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemColsB);
    }
}

// ---------------------------------------------------------------------------------------------
// dQ on tcgen05, query-major: a CTA owns one 128-row block (128/G queries x the G heads of a KV
// head) and walks the keys its rows see, 64 per step:
//   S  = Q K^T,  dP = dO V^T   (M = 128 rows, N = 64 keys)  -> TMEM, two buffers each (step & 1)
//   dS = P (dP - Drow), P = exp2(S scale_log2 - lse2)       by the compute warps (thread = row; the
//        row's lse, Drow and visible key range live in registers), 16-bit into a shared-memory
//        buffer of its own (step & 1)
//   dQ += dS K                 (A = dS from shared memory, B = K, MN-major) -> TMEM [256, 256 + D)
// The score products of a step go into the buffer the step before last used (its dS is already in
// shared memory), so they overlap the compute warps' work on the previous step; the dQ products come
// from a second issuing warp, so they run beside the next step's score products rather than queue
// behind them. The finished rows are scaled and written once.
//   warps 0..7  compute and the epilogue (two warps per 32 rows, each taking half of a step's keys
//               and of the dQ columns)
//   warp 8      loads: Q and dO of the block (TMA), the K and V rows of each step (TMA, one box per
//               page) into a ring of stages
//   warp 9      TMEM owner and issuer of the score products
//   warp 10     issuer of dQ += dS K (a second chain, which the tensor core overlaps with the first)
// ---------------------------------------------------------------------------------------------
namespace {

constexpr int QKB = 64;   // keys per step of the dQ kernel
constexpr int QKVST = 4;  // K/V stages (the fourth lets the loads run a step further ahead of dQ += dS K)
constexpr int kDqWarp = 10, kThreadsDq = 11 * 32;  // warp 10 issues dQ += dS K

template <int D>
struct BqCfg {
    static constexpr int KH = D / 64;
    static constexpr int HALF_R = 128 * 128;  // one 64-column half of the 128-row Q / dO tiles
    static constexpr int HALF_K = QKB * 128;  // one 64-column half of a 64-key K / V tile
    static constexpr int Q = 0;
    static constexpr int O = Q + KH * HALF_R;
    static constexpr int K = O + KH * HALF_R;                 // stage s: K at K + s * 2 * KH * HALF_K, V after
    static constexpr int DS = K + QKVST * 2 * KH * HALF_K;    // two dS buffers: 128 rows x 64 keys, 16-bit
    static constexpr int BAR = DS + 2 * 128 * 128;
    static constexpr int BYTES = BAR + 256;
    static constexpr int ALLOC = BYTES + 1024;
    static_assert(ALLOC <= 232448, "shared memory of one CTA");
    static constexpr int T_S = 0, T_DP = 128, T_DQ = 256;    // S_b at b * 64, dP_b at 128 + b * 64
    static constexpr int B_QFULL = 0, B_KVFULL = 1, B_KVEMPTY = B_KVFULL + QKVST, B_SFULL = B_KVEMPTY + QKVST,
                         B_PFULL = B_SFULL + 2, B_DSFREE = B_PFULL + 2, B_DQFULL = B_DSFREE + 2,
                         B_COUNT = B_DQFULL + 1;
};

}  // namespace

template <typename T, int D>
__global__ void __launch_bounds__(kThreadsDq, 1)
    bwd_tc_dq_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmo,
                     const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                     const BwdParams2 p) {
    using L_ = BqCfg<D>;
    constexpr int KH = L_::KH;
    constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
    constexpr uint32_t IDESC_S = idesc_f16(128, QKB, kBf16, false, false);
    constexpr uint32_t IDESC_DQ = idesc_f16(128, D, kBf16, false, true);

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L_::BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + L_::B_COUNT);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    const Watchdog wd{abort_flag, p.err, kWaitLimitNsB};

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const BwdRowUnit u = p.row_units[blockIdx.x];
    const int kvh = blockIdx.y;
    const SeqInfo si = p.seqs[u.seq];
    const int G = p.group;
    const int64_t base_pos = (int64_t)si.L - si.n;
    // keys any of the block's rows can see: [lo, hi), walked in steps of QKB from lo rounded down to
    // a multiple of QKB (so that every step starts on a page box)
    const int64_t p_first = base_pos + u.j0, p_last = base_pos + u.j1 - 1;
    const int64_t lo = (p.window > 0 ? max64(0, p_first - p.window + 1) : 0) / QKB * QKB;
    const int64_t hi = p.causal ? min64(si.L, p_last + 1) : si.L;
    const int nsteps = hi > lo ? (int)((hi - lo + QKB - 1) / QKB) : 0;
    const int ps = p.page_size, qbox = ps < QKB ? ps : QKB;  // rows of a K / V box
    // key rows of step j a box brings in: those of the boxes holding a key < hi; rows past that, or
    // past the sequence's end, hold arbitrary bytes (zeroed before dQ += dS K reads them)
    auto loaded_rows = [&](int j) {
        const int64_t t0 = lo + (int64_t)j * QKB;
        const int nb = (int)((min64(t0 + QKB, hi) - t0 + qbox - 1) / qbox);
        return (int)min64(nb * qbox, si.L - t0);
    };

    if (tid == 0) {
        for (int i = 0; i < L_::B_COUNT; ++i) {
            uint32_t cnt = 1;
            if (i == L_::B_PFULL || i == L_::B_PFULL + 1) cnt = kComputeWarpsB * 32;
            mbar_init(&bars[i], cnt);
        }
        *abort_flag = 0;
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(tmem_slot, kTmemColsB);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t s_base = smem_u32(smem);

    if (warp == kLoadWarp) {
        // ===================== loads =====================
        if (nsteps > 0 && lane == 0) {
            tma_prefetch(&tmq);
            tma_prefetch(&tmo);
            mbar_arrive_expect_tx(&bars[L_::B_QFULL], 2 * KH * L_::HALF_R);
            for (int h = 0; h < KH; ++h) {
                tma_load_3d(smem + L_::Q + h * L_::HALF_R, &tmq, &bars[L_::B_QFULL], h * 64, kvh * G,
                            si.q_start + u.j0);
                tma_load_3d(smem + L_::O + h * L_::HALF_R, &tmo, &bars[L_::B_QFULL], h * 64, kvh * G,
                            si.q_start + u.j0);
            }
        }
        // step j's K and V rows go into stage j % QKVST, one TMA box per page (and 64-column half)
        // holding a key < hi; lane l keeps the cache row of box base_g + l
        const int32_t* bt = p.block_tables + (int64_t)u.seq * p.table_width;
        const int bps = QKB / qbox;
        int base_g = -(1 << 30), my_row = 0;
        if (lane == 0) {
            tma_prefetch(&tmk);
            tma_prefetch(&tmv);
        }
        bool ok = true;
        for (int j = 0; ok && j < nsteps; ++j) {
            const int st = j % QKVST;
            const int64_t t0 = lo + (int64_t)j * QKB;
            const int nb = (int)((min64(t0 + QKB, hi) - t0 + qbox - 1) / qbox);
            const int g0 = j * bps;
            if (g0 + nb > base_g + 32) {
                base_g = g0;
                const int64_t key = lo + (int64_t)(base_g + lane) * qbox;
                my_row = key < si.L ? bt[key / ps] * ps + (int)(key % ps) : 0;
            }
            if (j >= QKVST)
                ok = __all_sync(0xffffffffu, mbar_wait(&bars[L_::B_KVEMPTY + st], ((j / QKVST) - 1) & 1, wd, 31));
            if (!ok) break;
            uint8_t* ks = smem + L_::K + st * 2 * KH * L_::HALF_K;
            uint8_t* vs = ks + KH * L_::HALF_K;
            if (lane == 0) mbar_arrive_expect_tx(&bars[L_::B_KVFULL + st], (uint32_t)(nb * qbox * 128 * KH * 2));
            for (int b = 0; b < nb; ++b) {
                const int row = __shfl_sync(0xffffffffu, my_row, g0 + b - base_g);
                if (lane == 0)
                    for (int h = 0; h < KH; ++h) {
                        tma_load_3d(ks + h * L_::HALF_K + b * qbox * 128, &tmk, &bars[L_::B_KVFULL + st], h * 64, kvh,
                                    row);
                        tma_load_3d(vs + h * L_::HALF_K + b * qbox * 128, &tmv, &bars[L_::B_KVFULL + st], h * 64, kvh,
                                    row);
                    }
            }
            __syncwarp();
        }
        if (lane == 0 && *abort_flag && nsteps > 0) {
            // leave no copy in flight into this CTA's shared memory (bounded, ignoring the flag)
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(&bars[L_::B_QFULL], 0) && globaltimer_ns() - t0 < kWaitLimitNsB) {}
            for (int j = max(0, nsteps - QKVST); j < nsteps; ++j)
                while (!mbar_try_wait(&bars[L_::B_KVFULL + j % QKVST], (j / QKVST) & 1) &&
                       globaltimer_ns() - t0 < kWaitLimitNsB) {}
        }
    } else if (warp == kMmaWarp) {
        // ===================== issuer of the score products =====================
        const uint64_t dQ = sdesc_sw128(s_base + L_::Q, 16, 1024);
        const uint64_t dO = sdesc_sw128(s_base + L_::O, 16, 1024);
        bool ok = nsteps == 0 || __all_sync(0xffffffffu, mbar_wait(&bars[L_::B_QFULL], 0, wd, 32));
        for (int j = 0; ok && j < nsteps; ++j) {
            const int st = j % QKVST, b = j & 1;
            // buffer b held S and dP of step j - 2, read by the compute warps before they marked P
            if (j >= 2) ok = __all_sync(0xffffffffu, mbar_wait(&bars[L_::B_PFULL + b], ((j - 2) >> 1) & 1, wd, 34));
            if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bars[L_::B_KVFULL + st], (j / QKVST) & 1, wd, 35));
            if (!ok) break;
            tc_fence_after();
            if (lane == 0) {
                const uint32_t ks = s_base + L_::K + st * 2 * KH * L_::HALF_K;
                const uint64_t dK = sdesc_sw128(ks, 16, 1024), dV = sdesc_sw128(ks + KH * L_::HALF_K, 16, 1024);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off_r = (kk >> 2) * L_::HALF_R + (kk & 3) * 32;
                    const uint32_t off_k = (kk >> 2) * L_::HALF_K + (kk & 3) * 32;
                    mma_f16_ss(tmem + L_::T_S + b * QKB, desc_add(dQ, off_r), desc_add(dK, off_k), IDESC_S, kk > 0);
                    mma_f16_ss(tmem + L_::T_DP + b * QKB, desc_add(dO, off_r), desc_add(dV, off_k), IDESC_S, kk > 0);
                }
                mma_commit(&bars[L_::B_SFULL + b]);
            }
            __syncwarp();
        }
    } else if (warp == kDqWarp) {
        // ===================== issuer of dQ += dS_j K_j =====================
        // dS of step j in buffer j & 1, K in stage j % QKVST; a chain of its own, so that the tensor
        // core runs it beside the next step's score products instead of behind them
        bool ok = true;
        for (int j = 0; ok && j < nsteps; ++j) {
            ok = __all_sync(0xffffffffu, mbar_wait(&bars[L_::B_PFULL + (j & 1)], (j >> 1) & 1, wd, 33));
            if (!ok) break;
            tc_fence_after();
            // K rows the step's boxes did not bring (or past the sequence's end) hold arbitrary bytes,
            // and dS is zero there: make them zero too, so that 0 * garbage cannot reach dQ. S and dP of
            // the step, which read them as well, are complete (the compute warps saw them before
            // marking P).
            const int nz = loaded_rows(j);
            if (nz < QKB) {
                uint8_t* ks = smem + L_::K + (j % QKVST) * 2 * KH * L_::HALF_K;
                for (int h = 0; h < KH; ++h) {
                    uint4* base = reinterpret_cast<uint4*>(ks + h * L_::HALF_K);
                    for (int c = nz * 8 + lane; c < QKB * 8; c += 32) base[c] = make_uint4(0u, 0u, 0u, 0u);
                }
                fence_proxy_async_smem();
                __syncwarp();
            }
            if (lane == 0) {
                const uint32_t ks = s_base + L_::K + (j % QKVST) * 2 * KH * L_::HALF_K;
                const uint64_t dA = sdesc_sw128(s_base + L_::DS + (j & 1) * 128 * 128, 16, 1024);
                const uint64_t dB = sdesc_sw128(ks, L_::HALF_K, 1024);  // K as (keys x D), MN-major
#pragma unroll
                for (int kk = 0; kk < QKB / 16; ++kk)
                    mma_f16_ss(tmem + L_::T_DQ, desc_add(dA, kk * 32), desc_add(dB, kk * 16 * 128), IDESC_DQ,
                               (j > 0 || kk > 0) ? 1u : 0u);
                mma_commit(&bars[L_::B_DSFREE + (j & 1)]);
                mma_commit(&bars[L_::B_KVEMPTY + j % QKVST]);
                if (j == nsteps - 1) mma_commit(&bars[L_::B_DQFULL]);
            }
            __syncwarp();
        }
    } else {
        // ===================== compute: thread = row, half hf of the keys / dQ columns =====================
        const int hf = warp >> 2;
        const int r = (warp & 3) * 32 + lane;
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        const int R = (u.j1 - u.j0) * G;  // live rows
        const bool live = r < R;
        const int64_t qrow = (int64_t)(si.q_start + u.j0 + (live ? r / G : 0)) * p.hq + kvh * G + (live ? r % G : 0);
        const float l = live ? p.lse[qrow] : neg_inf();
        const bool has = live && l != neg_inf();
        const float lse2 = has ? l * kLog2eB : 0.f;
        const float drow = has ? p.drow[qrow] : 0.f;
        const int64_t pos = base_pos + u.j0 + (live ? r / G : 0);
        const int64_t row_lo = has ? (p.window > 0 ? max64(0, pos - p.window + 1) : 0) : 0;
        const int64_t row_hi = has ? (p.causal ? min64(si.L, pos + 1) : si.L) : 0;
        uint8_t* dsbuf = smem + L_::DS;
        bool ok = true;
        for (int j = 0; j < nsteps; ++j) {
            const int b = j & 1;
            ok = __all_sync(0xffffffffu, mbar_wait(&bars[L_::B_SFULL + b], (j >> 1) & 1, wd, 36)) && ok;
            tc_fence_after();
            const int64_t t0 = lo + (int64_t)j * QKB;
            // columns outside [row_lo, row_hi) are masked: off_lo = t0 - row_lo, off_hi = t0 - row_hi
            const int off_lo = (int)max64(min64(t0 - row_lo, 1 << 20), -(1 << 20));
            const int off_hi = (int)max64(min64(t0 - row_hi, 1 << 20), -(1 << 20));
            uint32_t dk[16];
            {
                const int c = hf;  // keys 32 hf .. 32 hf + 31 of the step
                uint32_t sv[32], dv[32];
                tmem_ld32(tmem + L_::T_S + b * QKB + lane_off + c * 32, sv);
                tmem_ld32(tmem + L_::T_DP + b * QKB + lane_off + c * 32, dv);
                tmem_ld_wait(sv);
                tmem_regs_ready(dv);
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    float ds[2];
#pragma unroll
                    for (int x = 0; x < 2; ++x) {
                        const int k = c * 32 + 2 * e + x;
                        const bool vis = k + off_lo >= 0 && k + off_hi < 0;
                        const float pv = fast_exp2(fmaf(__uint_as_float(sv[2 * e + x]), p.scale_log2, -lse2));
                        ds[x] = vis ? pv * (__uint_as_float(dv[2 * e + x]) - drow) : 0.f;
                    }
                    dk[e] = pack2<T>(ds[0], ds[1]);
                }
            }
            // the dS buffer was last read by the dQ product of step j - 2
            if (j >= 2) ok = __all_sync(0xffffffffu, mbar_wait(&bars[L_::B_DSFREE + b], ((j - 2) >> 1) & 1, wd, 37)) && ok;
            // row r of dS: 64 keys = 128 bytes, 16-byte chunk ch at position ch ^ (r & 7); this warp
            // writes chunks 4 hf .. 4 hf + 3
            uint8_t* row = dsbuf + b * 128 * 128 + r * 128;
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4)
                *reinterpret_cast<uint4*>(row + (btc_swz(r, 4 * hf + q4) << 4)) =
                    make_uint4(dk[4 * q4], dk[4 * q4 + 1], dk[4 * q4 + 2], dk[4 * q4 + 3]);
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&bars[L_::B_PFULL + b]);
        }
        // ---- epilogue: the block's dQ rows, scaled, written once ----
        if (nsteps > 0 && ok) ok = __all_sync(0xffffffffu, mbar_wait(&bars[L_::B_DQFULL], 0, wd, 38));
        ok = __all_sync(0xffffffffu, ok);
        tc_fence_after();
        float* dst = p.dq + qrow * D;
#pragma unroll 1
        for (int c = hf * (D / 64); c < (hf + 1) * (D / 64); ++c) {
            uint32_t v[32];
            if (ok && nsteps > 0) {
                tmem_ld32(tmem + L_::T_DQ + lane_off + c * 32, v);
                tmem_ld_wait(v);
            } else {
#pragma unroll
                for (int e = 0; e < 32; ++e) v[e] = 0u;
            }
            if (live && ok) {
                float4* d4 = reinterpret_cast<float4*>(dst + c * 32);
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    d4[e] = make_float4(__uint_as_float(v[4 * e]) * p.scale, __uint_as_float(v[4 * e + 1]) * p.scale,
                                        __uint_as_float(v[4 * e + 2]) * p.scale, __uint_as_float(v[4 * e + 3]) * p.scale);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemColsB);
    }
}

namespace {

template <typename T, int D>
cudaError_t launch_btc(const BwdParams2& p, int num_key_units, int64_t num_queries, cudaStream_t st) {
    using L_ = BtcCfg<D>;
    const bool bf16 = std::is_same<T, __nv_bfloat16>::value;
    const int G = p.group, qpt = RB / G;
    const int ps = p.page_size;
    const uint64_t cache_rows = (uint64_t)p.num_pages * ps;
    // Q and dO: boxes of 128 rows (qpt queries x G heads) and 64 columns; K and V: one page (at
    // most the tile) of one KV head; the float32 gradient caches: 32 rows of one KV head
    CUtensorMap tq, to, tk, tv, tdk, tdv;
    if (!make_map(&tq, bf16, p.q, D, p.hq, (uint64_t)num_queries, G, qpt) ||
        !make_map(&to, bf16, p.dout, D, p.hq, (uint64_t)num_queries, G, qpt) ||
        !make_map(&tk, bf16, p.k, D, p.hkv, cache_rows, 1, ps < KT ? ps : KT) ||
        !make_map(&tv, bf16, p.v, D, p.hkv, cache_rows, 1, ps < KT ? ps : KT) ||
        !make_map_f32(&tdk, p.dk, D, p.hkv, cache_rows, 1, ps < 32 ? ps : 32) ||
        !make_map_f32(&tdv, p.dv, D, p.hkv, cache_rows, 1, ps < 32 ? ps : 32))
        return cudaErrorInvalidValue;
    auto kern = bwd_tc_dkdv_kernel<T, D>;
    static unsigned long long configured = 0;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 64 || !(configured >> dev & 1ull)) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L_::ALLOC);
        if (e != cudaSuccess) return e;
        if (dev < 64) configured |= 1ull << dev;
    }
    kern<<<dim3(num_key_units, p.hkv), kThreadsB, L_::ALLOC, st>>>(tq, to, tk, tv, tdk, tdv, p);
    return cudaGetLastError();
}

}  // namespace

template <typename T, int D>
cudaError_t launch_bq(const BwdParams2& p, int num_row_units, int64_t num_queries, cudaStream_t st) {
    using L_ = BqCfg<D>;
    const bool bf16 = std::is_same<T, __nv_bfloat16>::value;
    const int G = p.group, qpt = RB / G;
    const int ps = p.page_size;
    const uint64_t cache_rows = (uint64_t)p.num_pages * ps;
    CUtensorMap tq, to, tk, tv;  // Q, dO as in the dK/dV kernel; K, V: one page (at most a step) of a KV head
    if (!make_map(&tq, bf16, p.q, D, p.hq, (uint64_t)num_queries, G, qpt) ||
        !make_map(&to, bf16, p.dout, D, p.hq, (uint64_t)num_queries, G, qpt) ||
        !make_map(&tk, bf16, p.k, D, p.hkv, cache_rows, 1, ps < QKB ? ps : QKB) ||
        !make_map(&tv, bf16, p.v, D, p.hkv, cache_rows, 1, ps < QKB ? ps : QKB))
        return cudaErrorInvalidValue;
    auto kern = bwd_tc_dq_kernel<T, D>;
    static unsigned long long configured = 0;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 64 || !(configured >> dev & 1ull)) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L_::ALLOC);
        if (e != cudaSuccess) return e;
        if (dev < 64) configured |= 1ull << dev;
    }
    kern<<<dim3(num_row_units, p.hkv), kThreadsDq, L_::ALLOC, st>>>(tq, to, tk, tv, p);
    return cudaGetLastError();
}

int backward_tc_key_tile() { return KT; }
int backward_tc_row_block() { return RB; }

cudaError_t launch_backward_tc_dkdv(const BwdParams2& p, pa_dtype dt, int num_key_units, int64_t num_queries,
                                    cudaStream_t st) {
    if (num_key_units == 0) return cudaSuccess;
    if (dt == PA_BF16)
        return p.d == 64 ? launch_btc<__nv_bfloat16, 64>(p, num_key_units, num_queries, st)
                         : launch_btc<__nv_bfloat16, 128>(p, num_key_units, num_queries, st);
    return p.d == 64 ? launch_btc<__half, 64>(p, num_key_units, num_queries, st)
                     : launch_btc<__half, 128>(p, num_key_units, num_queries, st);
}


cudaError_t launch_backward_tc_dq(const BwdParams2& p, pa_dtype dt, int num_row_units, int64_t num_queries,
                                  cudaStream_t st) {
    if (num_row_units == 0) return cudaSuccess;
    if (dt == PA_BF16)
        return p.d == 64 ? launch_bq<__nv_bfloat16, 64>(p, num_row_units, num_queries, st)
                         : launch_bq<__nv_bfloat16, 128>(p, num_row_units, num_queries, st);
    return p.d == 64 ? launch_bq<__half, 64>(p, num_row_units, num_queries, st)
                     : launch_bq<__half, 128>(p, num_row_units, num_queries, st);
}

}  // namespace pa
