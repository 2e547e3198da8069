// Chunked-prefill paged attention on the 5th-generation tensor cores (tcgen05 + TMEM + TMA),
// bf16 / fp16, head_dim 64, 128 or 256, Dv == D.
//
// A unit is one 128-row tile: 128/G consecutive queries of a sequence times the G query heads
// that share one KV head (so every K/V tile feeds all G heads), against the keys those queries
// can see, BN keys per step (BN = 128; 64 at D = 256, where TMEM holds the two score buffers,
// the 256 output columns and the two P buffers only at that width); it ends with the final
// output and lse. The kernel is persistent:
// one CTA per SM walks the units in strides of the grid, and its pipelines run on from one unit
// into the next (the Q of the next unit loads as soon as the last score product of the current
// one has completed; K/V loads and score products of the next unit overlap the current unit's
// last softmax and output store).
//
//   warps 8, 11 TMA producers: warp 8 the Q tile once and the K tiles, warp 11 the V tiles, page
//               by page (one box per page and 64-element half of the head dim, 128-byte
//               swizzle) into rings of stages; pages past the sequence's last key are never
//               touched.
//   warp 9      TMEM owner and issuer (one thread) of S = Q K^T into one of two TMEM buffers.
//   warp 10     issuer (one thread) of O += P V with P read from TMEM; before it, the warp
//               zeroes the V rows past the sequence's last key (their bytes are whatever the page
//               holds there). Commits signal completion.
//   warps 0..7  softmax, two warps per row (each owning one half of the tile's columns; a warp's
//               lanes are the TMEM lanes of its quadrant): S from TMEM, scale to base-2
//               units, causal/window mask at absolute positions on edge tiles, running max and
//               sum in float32, P = exp2(S - m) packed to 16-bit into one of two TMEM P buffers.
//               Usually one pass with the running max; the output in TMEM is rescaled only when
//               the max grows by more than 2^8. The epilogue divides by the sum, rounds once
//               and stores.
//
// TMEM (512 columns): S0 [0,BN) S1 [BN,2BN) O [2BN,2BN+D) P0, P1 (BN/2 columns each) after O:
// 448 columns at D = 128 (BN 128) and at D = 256 (BN 64).
// QK of tile i+2 goes into score buffer i & 1 only after the softmax has marked P of tile i
// ready (it has then read all of S of tile i). The QK and the P V chains come from two issuing
// warps so that the tensor core overlaps them.
//
// Every wait on an mbarrier is bounded (Watchdog): a stalled pipeline sets the plan's error
// word and the CTA leaves through its normal exit, freeing TMEM.
#include <cudaTypedefs.h>

#include "sm100.cuh"

namespace pa {

using namespace sm100;

namespace {

constexpr int BM = 128;  // rows per tile (queries x group heads)
constexpr int kSoftmaxWarps = 8;  // two per TMEM lane quadrant, each owning half of the columns
constexpr int kTmaWarp = kSoftmaxWarps, kMmaWarp = kSoftmaxWarps + 1, kPvWarp = kSoftmaxWarps + 2;
constexpr int kTmaVWarp = kSoftmaxWarps + 3;  // the V producer (kTmaWarp loads Q and K)
constexpr int kThreads = (kSoftmaxWarps + 4) * 32;
constexpr uint32_t kTmemCols = 512;
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s: far beyond any legal wait

// Tile width and pipeline depth per head size. Shared memory: Q (D/64 boxes of 128 rows x
// 128 bytes) plus KST K and VST V stages of BN rows x D columns: 112 KB at D = 64, 224 KB at
// D = 128 (3 + 3 stages) and at D = 256 (64-key tiles, 3 + 2 stages), within the 227 KB of one
// CTA.
template <int D>
struct PrefillCfg {
    static constexpr int BN = D == 256 ? 64 : 128;  // keys per step
    static constexpr int KST = 3;                   // K stages
    static constexpr int VST = D == 256 ? 2 : 3;    // V stages
    static constexpr int NC = BN / 64;              // 32-column chunks of S per softmax warp
    static constexpr int KH = D / 64;               // 128-byte halves of a row
    static constexpr int HALF_Q = BM * 128;         // bytes of one half of the Q tile
    static constexpr int HALF_KV = BN * 128;        // bytes of one half of a K or V tile
    static constexpr int Q = 0;
    static constexpr int K = Q + KH * HALF_Q;
    static constexpr int V = K + KST * KH * HALF_KV;
    static constexpr int BAR = V + VST * KH * HALF_KV;
    // row statistics: slots of 128 rows x 2 column halves of float. Two alternating slots (one
    // barrier per exchange) at D = 64; at D = 128 and 256 one slot and two barriers per exchange,
    // which measured faster there (and the second slot's kilobyte does not fit beside 224 KB of
    // tiles and the alignment room).
    static constexpr int XSLOTS = D == 64 ? 2 : 1;
    static constexpr int XCH = BAR + 256;
    static constexpr int BYTES = XCH + XSLOTS * 2 * BM * 4;
    static constexpr int ALLOC = BYTES + 1024;        // room to align the base to 1024
    // TMEM columns: two score buffers, the output, two P buffers (16-bit pairs)
    static constexpr int T_S1 = BN, T_O = 2 * BN, T_P0 = 2 * BN + D, T_P1 = T_P0 + BN / 2;
    static_assert(T_P1 + BN / 2 <= 512, "TMEM holds S0, S1, O, P0 and P1");
    static_assert(ALLOC <= 232448, "shared memory of one CTA");
    // Barriers used once per tile in alternation come in pairs indexed by tile parity, so that no
    // waiter can ever find its barrier two phases ahead of the phase it waits for.
    static constexpr int B_QFULL = 0, B_KFULL = 1, B_KEMPTY = B_KFULL + KST, B_VFULL = B_KEMPTY + KST,
                         B_VEMPTY = B_VFULL + VST, B_SFULL = B_VEMPTY + VST, B_PFULL = B_SFULL + 2,
                         B_ODONE = B_PFULL + 2, B_QEMPTY = B_ODONE + 2, B_COUNT = B_QEMPTY + 1;
    static_assert(B_COUNT * 8 + 8 <= 256, "barriers, TMEM slot and abort flag fit their 256 bytes");
};

}  // namespace

// ---- softmax helpers: one thread owns one row of a score tile in TMEM ---------------------------
// Column c of the tile is masked when c + off_lo < 0 or c + off_hi >= 0, where off_lo = kt0 - row_lo
// and off_hi = kt0 - row_hi (the row's visible keys are [row_lo, row_hi)).

// Each helper covers the 32-column chunks [c0, c0 + NC): one half of the tile's columns.
template <int NC>
__device__ __forceinline__ float tile_max_full(uint32_t taddr, int c0) {
    float m0 = neg_inf(), m1 = neg_inf(), m2 = neg_inf(), m3 = neg_inf();
#pragma unroll 1
    for (int c = c0; c < c0 + NC; ++c) {
        uint32_t v[32];
        tmem_ld32(taddr + c * 32, v);
        tmem_ld_wait(v);
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
            m0 = fmaxf(m0, __uint_as_float(v[e]));
            m1 = fmaxf(m1, __uint_as_float(v[e + 1]));
            m2 = fmaxf(m2, __uint_as_float(v[e + 2]));
            m3 = fmaxf(m3, __uint_as_float(v[e + 3]));
        }
    }
    return fmaxf(fmaxf(m0, m1), fmaxf(m2, m3));
}

template <int NC>
__device__ __forceinline__ float tile_max_masked(uint32_t taddr, int c0, int off_lo, int off_hi) {
    float m0 = neg_inf(), m1 = neg_inf();
#pragma unroll 1
    for (int c = c0; c < c0 + NC; ++c) {
        uint32_t v[32];
        tmem_ld32(taddr + c * 32, v);
        tmem_ld_wait(v);
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
            const int k0 = c * 32 + e;
            const float x0 = (k0 + off_lo >= 0 && k0 + off_hi < 0) ? __uint_as_float(v[e]) : neg_inf();
            const float x1 = (k0 + 1 + off_lo >= 0 && k0 + 1 + off_hi < 0) ? __uint_as_float(v[e + 1]) : neg_inf();
            m0 = fmaxf(m0, x0);
            m1 = fmaxf(m1, x1);
        }
    }
    return fmaxf(m0, m1);
}

// Probabilities of columns 32c .. 32c+31 of a row, packed two per 32-bit word, go to TMEM
// columns 16c .. 16c+15 of the row's P buffer (the A operand layout of the P V MMA).
template <typename T, bool MASKED>
__device__ __forceinline__ float exp_chunk(const uint32_t (&v)[32], int c, float scale, float nm, uint32_t p_taddr,
                                           int off_lo, int off_hi) {
    uint32_t pk[16];
    float s0 = 0.f, s1 = 0.f;
#pragma unroll
    for (int e = 0; e < 16; ++e) {
        float x0 = __uint_as_float(v[2 * e]), x1 = __uint_as_float(v[2 * e + 1]);
        if (MASKED) {
            const int k0 = c * 32 + 2 * e;
            x0 = (k0 + off_lo >= 0 && k0 + off_hi < 0) ? x0 : neg_inf();
            x1 = (k0 + 1 + off_lo >= 0 && k0 + 1 + off_hi < 0) ? x1 : neg_inf();
        }
        const float a0 = fast_exp2(fmaf(x0, scale, nm));
        const float a1 = fast_exp2(fmaf(x1, scale, nm));
        s0 += a0;
        s1 += a1;
        pk[e] = pack2<T>(a0, a1);
    }
    tmem_st16(p_taddr + c * 16, pk);
    return s0 + s1;
}

// Second pass of the two-pass path: probabilities against the (new) row max m.
template <typename T, bool MASKED, int NC>
__device__ __forceinline__ float tile_exp(uint32_t taddr, int c0, float scale, float m, uint32_t p_taddr,
                                          int off_lo, int off_hi) {
    float sum = 0.f;
#pragma unroll 1
    for (int c = c0; c < c0 + NC; ++c) {
        uint32_t v[32];
        tmem_ld32(taddr + c * 32, v);
        tmem_ld_wait(v);
        sum += exp_chunk<T, MASKED>(v, c, scale, -m, p_taddr, off_lo, off_hi);
    }
    return sum;
}

// One pass with the row's running max m (known finite): probabilities relative to m go to the
// P buffer while the tile max of the raw scores is tracked; the caller keeps them when the max
// grew by at most 2^8 (so p <= 256), and otherwise redoes the tile.
template <typename T, bool MASKED>
__device__ __forceinline__ float tile_fused1(uint32_t taddr, int c0, float scale, float m, uint32_t p_taddr,
                                             int off_lo, int off_hi, float& m_raw) {
    uint32_t v0[32];
    tmem_ld32(taddr + c0 * 32, v0);
    tmem_ld_wait(v0);
    float m0 = neg_inf(), m1 = neg_inf();
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
        float x0 = __uint_as_float(v0[e]), x1 = __uint_as_float(v0[e + 1]);
        if (MASKED) {
            const int k0 = c0 * 32 + e;
            x0 = (k0 + off_lo >= 0 && k0 + off_hi < 0) ? x0 : neg_inf();
            x1 = (k0 + 1 + off_lo >= 0 && k0 + 1 + off_hi < 0) ? x1 : neg_inf();
        }
        m0 = fmaxf(m0, x0);
        m1 = fmaxf(m1, x1);
    }
    m_raw = fmaxf(m0, m1);
    return exp_chunk<T, MASKED>(v0, c0, scale, -m, p_taddr, off_lo, off_hi);
}

template <typename T, bool MASKED>
__device__ __forceinline__ float tile_fused2(uint32_t taddr, int c0, float scale, float m, uint32_t p_taddr,
                                             int off_lo, int off_hi, float& m_raw) {
    uint32_t v0[32], v1[32];
    tmem_ld32(taddr + c0 * 32, v0);  // both chunks in flight before the one wait
    tmem_ld32(taddr + (c0 + 1) * 32, v1);
    tmem_ld_wait(v0);
    tmem_regs_ready(v1);
    float m0 = neg_inf(), m1 = neg_inf();
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
        float x0 = __uint_as_float(v0[e]), x1 = __uint_as_float(v0[e + 1]);
        float y0 = __uint_as_float(v1[e]), y1 = __uint_as_float(v1[e + 1]);
        if (MASKED) {
            const int k0 = c0 * 32 + e, k1 = k0 + 32;
            x0 = (k0 + off_lo >= 0 && k0 + off_hi < 0) ? x0 : neg_inf();
            x1 = (k0 + 1 + off_lo >= 0 && k0 + 1 + off_hi < 0) ? x1 : neg_inf();
            y0 = (k1 + off_lo >= 0 && k1 + off_hi < 0) ? y0 : neg_inf();
            y1 = (k1 + 1 + off_lo >= 0 && k1 + 1 + off_hi < 0) ? y1 : neg_inf();
        }
        m0 = fmaxf(m0, fmaxf(x0, y0));
        m1 = fmaxf(m1, fmaxf(x1, y1));
    }
    m_raw = fmaxf(m0, m1);
    return exp_chunk<T, MASKED>(v0, c0, scale, -m, p_taddr, off_lo, off_hi) +
           exp_chunk<T, MASKED>(v1, c0 + 1, scale, -m, p_taddr, off_lo, off_hi);
}

template <typename T, bool MASKED, int NC>
__device__ __forceinline__ float tile_fused(uint32_t taddr, int c0, float scale, float m, uint32_t p_taddr,
                                            int off_lo, int off_hi, float& m_raw) {
    if constexpr (NC == 1) return tile_fused1<T, MASKED>(taddr, c0, scale, m, p_taddr, off_lo, off_hi, m_raw);
    else return tile_fused2<T, MASKED>(taddr, c0, scale, m, p_taddr, off_lo, off_hi, m_raw);
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                      const __grid_constant__ CUtensorMap tmv, const AttnParams p) {
    using L_ = PrefillCfg<D>;
    constexpr int KH = L_::KH, BN = L_::BN, KST = L_::KST, VST = L_::VST, NC = L_::NC;
    constexpr int B_QFULL = L_::B_QFULL, B_KFULL = L_::B_KFULL, B_KEMPTY = L_::B_KEMPTY, B_VFULL = L_::B_VFULL,
                  B_VEMPTY = L_::B_VEMPTY, B_SFULL = L_::B_SFULL, B_PFULL = L_::B_PFULL, B_ODONE = L_::B_ODONE,
                  B_QEMPTY = L_::B_QEMPTY, B_COUNT = L_::B_COUNT;
    constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
    constexpr uint32_t IDESC_QK = idesc_f16(BM, BN, kBf16, false, false);
    constexpr uint32_t IDESC_PV = idesc_f16(BM, D, kBf16, false, true);

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L_::BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + B_COUNT);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    const Watchdog wd{abort_flag, p.err, kWaitLimitNs};

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = p.group;
    const int qpt = BM / G;
    const int ps = p.page_size;
    const int box = ps < BN ? ps : BN;  // keys per TMA box

    if (tid == 0) {
        for (int i = 0; i < B_COUNT; ++i) {
            uint32_t cnt = 1;
            if (i == B_PFULL || i == B_PFULL + 1) cnt = kSoftmaxWarps * 32;
            mbar_init(&bars[i], cnt);
        }
        *abort_flag = 0;
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t t_s0 = tmem, t_s1 = tmem + L_::T_S1;
    const uint32_t t_o = tmem + L_::T_O;
    const uint32_t t_p0 = tmem + L_::T_P0, t_p1 = tmem + L_::T_P1;
    const uint32_t s_base = smem_u32(smem);

    // Units come longest first from the host. In round rr the CTA takes unit rr * grid + b, with b
    // = blockIdx.x on even rounds and grid - 1 - blockIdx.x on odd ones (a snake over the sorted
    // list keeps the work per CTA even). Every role walks the same sequence and counts the key
    // tiles it has passed (gt) and the units with at least one tile (kq); stage indices and
    // barrier phases follow those running counts across units.
    const int rounds = (p.num_punits + (int)gridDim.x - 1) / (int)gridDim.x;
    auto unit_of = [&](int rr) {
        return rr * (int)gridDim.x + ((rr & 1) ? (int)gridDim.x - 1 - (int)blockIdx.x : (int)blockIdx.x);
    };
    auto view_of = [&](int ui, PrefillUnit& u, SeqInfo& si, int& live_q, int64_t& p_first, int64_t& kt_start,
                       int& n_tiles) {
        u = p.punits[ui];
        si = p.seqs[u.seq];
        live_q = min(qpt, si.n - u.j0);
        p_first = (int64_t)si.L - si.n + u.j0;
        const int64_t p_last = p_first + live_q - 1;
        const int64_t kv_lo = p.window > 0 ? max64(0, p_first - p.window + 1) : 0;
        const int64_t kv_hi = p.causal ? min64(si.L, p_last + 1) : si.L;
        kt_start = (kv_lo / box) * box;
        n_tiles = kv_hi > kt_start ? (int)((kv_hi - kt_start + BN - 1) / BN) : 0;
    };

    if (warp == kTmaWarp || warp == kTmaVWarp) {
        // ===================== TMA producers =====================
        // One warp loads Q and the K tiles, another the V tiles, so that neither waits for the
        // other's stages. The whole warp runs the loop; lane 0 issues. Page ids of the next 32
        // boxes are read from the block table by the 32 lanes at once and handed to lane 0 by
        // shuffles, so a table read never sits between two loads.
        const bool is_v = warp == kTmaVWarp;
        const int NST = is_v ? VST : KST;
        const CUtensorMap* tm = is_v ? &tmv : &tmk;
        uint64_t* full = &bars[is_v ? B_VFULL : B_KFULL];
        uint64_t* empty = &bars[is_v ? B_VEMPTY : B_KEMPTY];
        uint8_t* ring = smem + (is_v ? L_::V : L_::K);
        if (lane == 0) {
            tma_prefetch(tm);
            if (!is_v) tma_prefetch(&tmq);
        }
        const int bpt = BN / box;  // boxes per tile (<= 8)
        int gt = 0, kq = 0;        // tiles and Q tiles issued
        bool ok = true;
        for (int rr = 0; ok && rr < rounds; ++rr) {
            const int ui = unit_of(rr);
            if (ui >= p.num_punits) continue;
            PrefillUnit u;
            SeqInfo si;
            int live_q, n_tiles;
            int64_t p_first, kt_start;
            view_of(ui, u, si, live_q, p_first, kt_start, n_tiles);
            if (n_tiles == 0) continue;
            if (!is_v) {
                // the Q buffer is free once every S = Q K^T of the previous unit has completed
                if (kq > 0 && !__all_sync(0xffffffffu, mbar_wait(&bars[B_QEMPTY], (kq - 1) & 1, wd, 12))) break;
                if (lane == 0) {
                    mbar_arrive_expect_tx(&bars[B_QFULL], KH * L_::HALF_Q);
                    for (int h = 0; h < KH; ++h)
                        tma_load_3d(smem + L_::Q + h * L_::HALF_Q, &tmq, &bars[B_QFULL], h * 64, u.kvh * G,
                                    si.q_start + u.j0);
                }
            }
            ++kq;
            const int32_t* bt = p.block_tables + (int64_t)u.seq * p.table_width;
            int base_g = -(1 << 30);  // first box whose page id the lanes hold
            int my_row = 0;           // lane l: first cache row of box base_g + l
            for (int i = 0; i < n_tiles; ++i, ++gt) {
                const int64_t kt0 = kt_start + (int64_t)i * BN;
                int nb = 0;  // boxes whose first key lies inside the sequence
                for (int b = 0; b < bpt; ++b)
                    if (kt0 + (int64_t)b * box < si.L) nb = b + 1;
                const int g0 = i * bpt;
                if (g0 + nb > base_g + 32) {
                    base_g = g0;
                    const int64_t key = kt_start + (int64_t)(base_g + lane) * box;
                    my_row = key < si.L ? (int)((int64_t)bt[key / ps] * ps + key % ps) : 0;
                }
                const int st = gt % NST;
                if (gt >= NST && !__all_sync(0xffffffffu, mbar_wait(empty + st, ((gt / NST) - 1) & 1, wd, is_v ? 2 : 1))) {
                    ok = false;
                    break;
                }
                if (lane == 0) mbar_arrive_expect_tx(full + st, (uint32_t)nb * box * 128 * KH);
                for (int b = 0; b < nb; ++b) {
                    const int row = __shfl_sync(0xffffffffu, my_row, g0 + b - base_g);
                    if (lane == 0)
                        for (int h = 0; h < KH; ++h)
                            tma_load_3d(ring + (st * KH + h) * L_::HALF_KV + b * box * 128, tm, full + st, h * 64,
                                        u.kvh, row);
                }
            }
        }
        if (lane == 0 && *abort_flag) {
            // Leave no copy in flight into this CTA's shared memory: wait (bounded, ignoring the
            // abort flag) for the last loads issued into each stage (and for the last Q).
            const uint64_t t0 = globaltimer_ns();
            auto drain = [&](uint64_t* bar, uint32_t parity) {
                while (!mbar_try_wait(bar, parity) && globaltimer_ns() - t0 < kWaitLimitNs) {}
            };
            if (!is_v && kq > 0) drain(&bars[B_QFULL], (kq - 1) & 1);
            for (int i = max(0, gt - NST); i < gt; ++i) drain(full + i % NST, (i / NST) & 1);
        }
    } else if (warp == kMmaWarp || warp == kPvWarp) {
        // ===================== MMA issuers =====================
        // Two warps issue: one the S = Q K^T chains, one the O += P V chains. The tensor core
        // runs the MMAs of one issuing warp one after the other, each k-step paying a latency
        // well above its throughput (about twice as much for the TMEM-operand form of P V);
        // chains from two warps overlap. Descriptors are built once; a k-step or stage offset
        // is an add to the address field.
        const uint64_t dQ = sdesc_sw128(s_base + L_::Q, 16, 1024);
        const uint64_t dK = sdesc_sw128(s_base + L_::K, 16, 1024);
        const uint64_t dV = sdesc_sw128(s_base + L_::V, L_::HALF_KV, 1024);
        int gt = 0, kq = 0;
        bool ok = true;
        for (int rr = 0; ok && rr < rounds; ++rr) {
            const int ui = unit_of(rr);
            if (ui >= p.num_punits) continue;
            PrefillUnit u;
            SeqInfo si;
            int live_q, n_tiles;
            int64_t p_first, kt_start;
            view_of(ui, u, si, live_q, p_first, kt_start, n_tiles);
            if (n_tiles == 0) continue;
            if (warp == kMmaWarp) {
                // S of tile gt goes into score buffer gt & 1, free again once the softmax has
                // marked P of tile gt - 2 ready (it has then read all of S of that tile).
                ok = __all_sync(0xffffffffu, mbar_wait(&bars[B_QFULL], kq & 1, wd, 3));
                for (int i = 0; ok && i < n_tiles; ++i, ++gt) {
                    const int ks = gt % KST, b = gt & 1;
                    if (gt >= 2) ok = __all_sync(0xffffffffu, mbar_wait(&bars[B_PFULL + b], ((gt - 2) >> 1) & 1, wd, 6));
                    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bars[B_KFULL + ks], (gt / KST) & 1, wd, 4));
                    if (!ok) break;
                    tc_fence_after();
                    if (lane == 0) {
                        const uint32_t d_s = b ? t_s1 : t_s0;
                        const uint64_t dKs = desc_add(dK, ks * KH * L_::HALF_KV);
#pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk) {
                            // k-step kk: 128-byte half kk / 4 of the rows, 32-byte slice kk % 4 of it
                            const uint32_t off_q = (kk >> 2) * L_::HALF_Q + (kk & 3) * 32;
                            const uint32_t off_k = (kk >> 2) * L_::HALF_KV + (kk & 3) * 32;
                            mma_f16_ss(d_s, desc_add(dQ, off_q), desc_add(dKs, off_k), IDESC_QK, kk > 0);
                        }
                        mma_commit(&bars[B_SFULL + b]);
                        mma_commit(&bars[B_KEMPTY + ks]);
                        if (i == n_tiles - 1) mma_commit(&bars[B_QEMPTY]);
                    }
                    __syncwarp();
                }
            } else {
                // O += P V of tile gt once P of that tile and its V tile are in place; the first
                // tile of a unit starts O afresh (the softmax has read the previous unit's O
                // before it marks that P ready).
                for (int j = 0; ok && j < n_tiles; ++j, ++gt) {
                    const int vs = gt % VST;
                    ok = __all_sync(0xffffffffu, mbar_wait(&bars[B_PFULL + (gt & 1)], (gt >> 1) & 1, wd, 6));
                    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bars[B_VFULL + vs], (gt / VST) & 1, wd, 7));
                    if (!ok) break;
                    // V rows past the sequence's end hold arbitrary bytes: make them zero.
                    const int64_t kt0 = kt_start + (int64_t)j * BN;
                    const int nvalid = (int)min64(BN, si.L - kt0);
                    if (nvalid < BN) {
                        for (int h = 0; h < KH; ++h) {
                            uint4* base = reinterpret_cast<uint4*>(smem + L_::V + (vs * KH + h) * L_::HALF_KV);
                            for (int c = nvalid * 8 + lane; c < BN * 8; c += 32) base[c] = make_uint4(0, 0, 0, 0);
                        }
                        fence_proxy_async_smem();
                        __syncwarp();
                    }
                    tc_fence_after();
                    if (lane == 0) {
                        const uint32_t t_pj = (gt & 1) ? t_p1 : t_p0;
                        const uint64_t dVs = desc_add(dV, vs * KH * L_::HALF_KV);
                        const uint32_t acc0 = j > 0 ? 1u : 0u;
#pragma unroll
                        for (int kk = 0; kk < BN / 16; ++kk)  // 16 keys = 8 TMEM columns of P
                            mma_f16_ts(t_o, t_pj + kk * 8, desc_add(dVs, kk * 16 * 128), IDESC_PV, kk > 0 ? 1u : acc0);
                        mma_commit(&bars[B_ODONE + (gt & 1)]);
                        mma_commit(&bars[B_VEMPTY + vs]);
                    }
                    __syncwarp();
                }
            }
            ++kq;
        }
    } else {
        // ===================== softmax: thread = row, two warps per row =====================
        // Warp w owns TMEM lanes 32(w % 4) .. +31 (its rows) and columns half (w / 4) of every
        // tile; the two warps of a row keep identical running maxima, exchange their partial
        // maxima through shared memory when needed and add their partial sums at the end.
        const int quad = warp & 3, half = warp >> 2;
        const int r = quad * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        const int c0 = half * NC;  // first 32-column chunk of this warp's half
        float* xch = reinterpret_cast<float*>(smem + L_::XCH);
        auto pair_sync = [&]() { asm volatile("bar.sync %0, 64;\n" ::"r"(1 + quad) : "memory"); };
        // max (or sum) of this row's two halves. Both warps of a row make the same exchanges in the
        // same order. With two slots exchange x uses slot x & 1, so a slot is written again only
        // after the next exchange's barrier, which the partner reaches after reading it: one
        // barrier each. With one slot a second barrier keeps the next write behind the partner's read.
        uint32_t n_xch = 0;
        auto exchange = [&](float mine, bool is_max) {
            float* slot = xch + (L_::XSLOTS == 2 ? (n_xch++ & 1u) * 2 * BM : 0u);
            slot[half * BM + r] = mine;
            pair_sync();
            const float other = slot[(1 - half) * BM + r];
            if (L_::XSLOTS == 1) pair_sync();
            return is_max ? fmaxf(mine, other) : mine + other;
        };
        int gt = 0;
        bool ok = true;
        // After an abort the loops still run to their ends (every wait then returns at once), so
        // that both warps of a row reach the same row-statistics exchanges.
        for (int rr = 0; rr < rounds; ++rr) {
            const int ui = unit_of(rr);
            if (ui >= p.num_punits) continue;
            PrefillUnit u;
            SeqInfo si;
            int live_q, n_tiles;
            int64_t p_first, kt_start;
            view_of(ui, u, si, live_q, p_first, kt_start, n_tiles);
            const int live_rows = live_q * G;
            const int64_t p_last = p_first + live_q - 1;
            const bool live = r < live_rows;
            const int64_t pos = p_first + (live ? r / G : 0);
            // keys this row sees: [row_lo, row_hi) (padding rows: every key of the sequence)
            const int64_t row_lo = (live && p.window > 0) ? max64(0, pos - p.window + 1) : 0;
            const int64_t row_hi = (live && p.causal) ? min64(si.L, pos + 1) : si.L;
            // keys every live row sees: [all_lo, all_hi)
            const int64_t all_lo = p.window > 0 ? p_last - p.window + 1 : INT64_MIN;
            const int64_t all_hi = min64(p.causal ? p_first + 1 : si.L, si.L);
            float m_run = neg_inf(), l_part = 0.f;
            for (int i = 0; i < n_tiles; ++i, ++gt) {
                const int b = gt & 1;
                const int64_t kt0 = kt_start + (int64_t)i * BN;
                const uint32_t t_sb = (b ? t_s1 : t_s0) + lane_off;
                const bool full = kt0 >= all_lo && kt0 + BN <= all_hi;
                ok = __all_sync(0xffffffffu, mbar_wait(&bars[B_SFULL + b], (gt >> 1) & 1, wd, 8)) && ok;
                tc_fence_after();
                // P buffer b was last read by P V of tile gt - 2
                if (gt >= 2) {
                    ok = __all_sync(0xffffffffu, mbar_wait(&bars[B_ODONE + b], ((gt - 2) >> 1) & 1, wd, 11)) && ok;
                }
                const uint32_t t_pb = (b ? t_p1 : t_p0) + lane_off;
                const int off_lo = (int)(kt0 - row_lo), off_hi = (int)(kt0 - row_hi);
                // Fast path: one pass with the running max when every row of the warp has one (both
                // warps of a row decide alike: their running maxima are equal).
                bool redo = true;
                float sum = 0.f;
                if (__all_sync(0xffffffffu, m_run != neg_inf())) {
                    float m_raw;
                    sum = full ? tile_fused<T, false, NC>(t_sb, c0, p.scale_log2, m_run, t_pb, 0, 0, m_raw)
                               : tile_fused<T, true, NC>(t_sb, c0, p.scale_log2, m_run, t_pb, off_lo, off_hi, m_raw);
                    m_raw = exchange(m_raw, true);
                    redo = __any_sync(0xffffffffu, m_raw * p.scale_log2 > m_run + 8.0f);
                }
                if (redo) {
                    // pass 1: tile max of the raw scores; the scale is positive, so it is applied to
                    // the max once. Edge tiles mask keys outside [row_lo, row_hi) first.
                    float m_raw = full ? tile_max_full<NC>(t_sb, c0) : tile_max_masked<NC>(t_sb, c0, off_lo, off_hi);
                    m_raw = exchange(m_raw, true);
                    const float m_tile = m_raw * p.scale_log2;
                    const float m_new = fmaxf(m_run, m_tile);
                    const bool grow = m_new > m_run + 8.0f;  // also true when m_run is -inf and m_new finite
                    const bool rescale = grow && i > 0 && m_run != neg_inf();
                    if (__any_sync(0xffffffffu, rescale)) {
                        // the output must hold every earlier tile of the unit before it is rescaled
                        ok = __all_sync(0xffffffffu, mbar_wait(&bars[B_ODONE + ((gt - 1) & 1)], ((gt - 1) >> 1) & 1, wd, 9)) && ok;
                        tc_fence_after();
                        const float alpha = rescale ? fast_exp2(m_run - m_new) : 1.0f;
#pragma unroll 1
                        for (int c = half * (D / 64); c < (half + 1) * (D / 64); ++c) {  // this warp's half of O
                            uint32_t v[32];
                            tmem_ld32(t_o + lane_off + c * 32, v);
                            tmem_ld_wait(v);
#pragma unroll
                            for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * alpha);
                            tmem_st32(t_o + lane_off + c * 32, v);
                        }
                    }
                    if (grow) {
                        l_part *= fast_exp2(m_run - m_new);
                        m_run = m_new;
                    }
                    const float m_use = m_run == neg_inf() ? 0.f : m_run;
                    // pass 2: probabilities p = 2^(s * scale - m) into the P buffer
                    sum = full ? tile_exp<T, false, NC>(t_sb, c0, p.scale_log2, m_use, t_pb, 0, 0)
                               : tile_exp<T, true, NC>(t_sb, c0, p.scale_log2, m_use, t_pb, off_lo, off_hi);
                }
                tmem_st_wait();
                l_part += sum;
                tc_fence_before();
                mbar_arrive(&bars[B_PFULL + b]);
            }
            // ---- epilogue: each warp of the pair stores its half of the output columns ----
            if (ok && n_tiles > 0)
                ok = __all_sync(0xffffffffu,
                                mbar_wait(&bars[B_ODONE + ((gt - 1) & 1)], ((gt - 1) >> 1) & 1, wd, 10));
            ok = __all_sync(0xffffffffu, ok);
            const float l_run = exchange(l_part, false);
            tc_fence_after();
            const bool has = l_run > 0.f;
            const float inv = has ? 1.0f / l_run : 0.f;
            const int64_t qrow = (int64_t)(si.q_start + u.j0 + (live ? r / G : 0)) * p.hq + u.kvh * G + (live ? r % G : 0);
            T* orow = static_cast<T*>(p.out) + qrow * D;
#pragma unroll 1
            for (int c = half * (D / 64); c < (half + 1) * (D / 64); ++c) {
                uint32_t v[32];
                if (ok && n_tiles > 0) {
                    tmem_ld32(t_o + lane_off + c * 32, v);
                    tmem_ld_wait(v);
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) v[e] = 0u;
                }
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    pk[e] = pack2<T>(__uint_as_float(v[2 * e]) * inv, __uint_as_float(v[2 * e + 1]) * inv);
                if (live && ok) {
                    uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
                    for (int e = 0; e < 4; ++e) dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
                }
            }
            if (live && ok && half == 0) p.lse[qrow] = has ? (m_run + __log2f(l_run)) * kLn2 : neg_inf();
            // the next unit's first P V overwrites O: this warp's reads of it are complete
            tc_fence_before();
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ---------------------------------------------------------------------------------------------
// Host side: tensor maps and launch
// ---------------------------------------------------------------------------------------------
namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

}  // namespace

// 3-D map over a row-major [d2][d1][d0] tensor of 16-bit elements, box {64, b1, b2}, 128B swizzle.
bool make_map(CUtensorMap* m, bool bf16, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t b1,
              uint32_t b2) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {d0, d1, d2};
    cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};
    cuuint32_t boxd[3] = {64, b1, b2};
    cuuint32_t es[3] = {1, 1, 1};
    CUresult r = fn(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3,
                    const_cast<void*>(base), dims, strides, boxd, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool make_map_f32(CUtensorMap* m, const float* base, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t b1, uint32_t b2) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {d0, d1, d2};
    cuuint64_t strides[2] = {d0 * 4, d0 * d1 * 4};
    cuuint32_t boxd[3] = {32, b1, b2};
    cuuint32_t es[3] = {1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(base), dims, strides, boxd, es,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

namespace {

template <typename T, int D>
cudaError_t launch_t(const AttnParams& p, int num_pages, cudaStream_t st) {
    using L_ = PrefillCfg<D>;
    constexpr int BN = L_::BN;
    const bool bf16 = std::is_same<T, __nv_bfloat16>::value;
    const int G = p.group, qpt = BM / G;
    const int ps = p.page_size;
    const int box = ps < BN ? ps : BN;
    CUtensorMap tq, tk, tv;  // the Q map spans every packed query row
    if (!make_map(&tq, bf16, p.q, D, p.hq, (uint64_t)p.num_queries, G, qpt) ||
        !make_map(&tk, bf16, p.k, D, p.hkv, (uint64_t)num_pages * ps, 1, box) ||
        !make_map(&tv, bf16, p.v, D, p.hkv, (uint64_t)num_pages * ps, 1, box))
        return cudaErrorInvalidValue;
    auto kern = prefill_tc_kernel<T, D>;
    static unsigned long long configured = 0;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 64 || !(configured >> dev & 1ull)) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L_::ALLOC);
        if (e != cudaSuccess) return e;
        if (dev < 64) configured |= 1ull << dev;
    }
    // persistent: one CTA per SM (shared memory allows no more), each walking units in strides
    static int sms[64] = {0};
    int nsm = dev < 64 ? sms[dev] : 0;
    if (nsm == 0) {
        e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
        if (dev < 64) sms[dev] = nsm;
    }
    const int grid = p.num_punits < nsm ? p.num_punits : nsm;
    kern<<<grid, kThreads, L_::ALLOC, st>>>(tq, tk, tv, p);
    return cudaGetLastError();
}

}  // namespace

bool prefill_tc_supported(pa_dtype dt, int d, int dv, int group, int page_size) {
    if (dt == PA_F32 || d != dv || (d != 64 && d != 128 && d != 256)) return false;
    if (group < 1 || group > BM || BM % group != 0) return false;
    if (page_size % 16 != 0) return false;
    const int bn = d == 256 ? PrefillCfg<256>::BN : PrefillCfg<128>::BN;  // a page box holds whole tiles, or a tile whole pages
    if (page_size < bn ? (bn % page_size != 0) : (page_size % bn != 0)) return false;
    return true;
}

template <typename T>
cudaError_t launch_d(const AttnParams& p, int num_pages, cudaStream_t st) {
    if (p.d == 64) return launch_t<T, 64>(p, num_pages, st);
    if (p.d == 256) return launch_t<T, 256>(p, num_pages, st);
    return launch_t<T, 128>(p, num_pages, st);
}

cudaError_t launch_prefill_tc(const AttnParams& p, pa_dtype dt, int num_pages, cudaStream_t st) {
    if (p.num_punits == 0) return cudaSuccess;
    if (dt == PA_BF16) return launch_d<__nv_bfloat16>(p, num_pages, st);
    return launch_d<__half>(p, num_pages, st);
}

}  // namespace pa
