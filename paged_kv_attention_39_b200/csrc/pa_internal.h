// Internal types shared by the host plan code and the kernels of libpa.so.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "pa.h"

namespace pa {

// Per-sequence facts on the device (16 bytes).
struct SeqInfo {
    int32_t L;        // keys in the cache, including the sequence's own new keys
    int32_t q_start;  // first packed query row
    int32_t n;        // number of queries
    int32_t pad;
};

// One unit of key-split work on the decode-style kernels: queries j0 .. j1-1 of sequence
// `seq` against keys [t0, t1) (the union of what those queries can see, cut into parts), for
// the KV head given by blockIdx.y. nsplit == 1 means the unit writes final results;
// otherwise query j's part `split` goes to workspace slot
// part_base + (j - j0) * nsplit + split.
struct KvUnit {
    int32_t seq, t0, t1, split;
    int32_t nsplit, part_base, j0, j1;
};

// One query row set to merge: query `query`, parts part_base .. part_base + nsplit - 1.
struct CombineUnit {
    int32_t query, part_base, nsplit, pad;
};

// One prefill tile: queries [j0, j0 + qpt) of sequence `seq` (qpt = 128 / G rows), keys
// [t0, t1), KV head kvh.
struct PrefillUnit {
    int32_t seq, j0, t0, t1;
    int32_t kvh, pad0, pad1, pad2;
};

// Backward on the tensor cores: a 128-key tile of sequence `seq` starting at key k0 (dK/dV
// kernel), and queries j0 .. j1-1 of a sequence, at most 128 rows per KV head (dQ kernel).
// ord >= 0: the tile touches a page that another key of the plan shares; its finished rows go
// to scratch tile `ord` and the ordered pass adds them (in sequence order) instead of the tile.
struct BwdKeyUnit {
    int32_t seq, k0, ord, pad;
};
// Ordered pass: cache row `slot` (page * page_size + slot in page) receives the scratch rows
// refs[begin .. begin + count) (scratch tile * 64 + row), summed in that order.
struct BwdSlotSum {
    int64_t slot;
    int32_t begin, count;
};
struct BwdRowUnit {
    int32_t seq, j0, j1, pad;
};

struct BwdParams2 {
    const void* q;       // [Nq, Hq, D]
    const void* k;       // [P, ps, Hkv, D]
    const void* v;       // [P, ps, Hkv, D]
    const void* out;     // [Nq, Hq, D] forward output
    const float* lse;    // [Nq, Hq] forward logsumexp (natural log)
    const void* dout;    // [Nq, Hq, D]
    float* drow;         // [Nq, Hq] dO . O, written by the first kernel
    float* dq;           // [Nq, Hq, D] written
    float* dk;           // [P, ps, Hkv, D] added into
    float* dv;           // [P, ps, Hkv, D] added into
    const SeqInfo* seqs;
    const int32_t* block_tables;
    const BwdKeyUnit* key_units;
    const BwdRowUnit* row_units;
    float* scratch_k;             // [ordered tiles, Hkv, 64, D] finished rows of ordered tiles
    float* scratch_v;
    const BwdSlotSum* slot_sums;  // ordered pass work list
    const int32_t* slot_refs;
    int32_t table_width, page_size, hq, hkv, group, d;
    float scale, scale_log2;
    int32_t causal, window;
    int32_t num_pages;
    int* err;  // device error word of the plan (bounded waits of the tcgen05 kernel)
};

// Everything a kernel needs; passed by value.
struct AttnParams {
    const void* q;    // [Nq, Hq, D]   (MLA: absorbed q [Nq, H, R])
    const void* k;    // [P, ps, Hkv, D] (MLA: latent [P, ps, 1, R])
    const void* v;    // [P, ps, Hkv, Dv] (MLA: same as k)
    const void* qr;   // MLA only: position q [Nq, H, Pr]
    const void* kr;   // MLA only: rope cache [P, ps, 1, Pr]
    void* out;        // [Nq, Hq, Dv]
    float* lse;       // [Nq, Hq]
    float* ws_o;      // [slots, Hq, Dv] float32 split partials (normalised)
    float* ws_lse;    // [slots, Hq] float32 (natural log)
    const SeqInfo* seqs;
    const int32_t* block_tables;
    const KvUnit* units;
    const CombineUnit* cunits;
    const PrefillUnit* punits;
    int32_t num_units, num_cunits, num_punits;
    int32_t table_width, page_size;
    int32_t hq, hkv, group, d, dv, pr;
    float scale;       // softmax scale
    float scale_log2;  // scale * log2(e): scores in base-2 units
    int32_t causal, window;
    int32_t num_queries, num_pages;
    int* err;          // device error word of the plan (0 = no failure)
    // Sparse top-K attention: when sel is set, a unit's keys [t0, t1) are positions in the
    // concatenation of the row's selected blocks: key v is position sel[row][v / block_size] *
    // block_size + v % block_size of the sequence (entries of -1 hold no keys).
    const int32_t* sel;  // [Nq, Hkv, sel_width] checked, compacted selection
    int32_t sel_width, block_size;
    // Tensor-core decode only: when set, split rows are merged by the kernel itself: the CTA that
    // finishes a (row set, KV head) last, counted at merge_ctr[part_base * hkv + kvh], merges its
    // parts and puts the counter back to zero (the counters are zero between calls).
    int* merge_ctr;
};

// Kernel launchers (one per .cu file). Each returns the launch's cudaError_t.
cudaError_t launch_simt(const AttnParams& p, pa_dtype dt, cudaStream_t st);
cudaError_t launch_decode_mma(const AttnParams& p, pa_dtype dt, int rows_max, cudaStream_t st);
cudaError_t launch_combine(const AttnParams& p, pa_dtype dt, cudaStream_t st);
cudaError_t launch_prefill_tc(const AttnParams& p, pa_dtype dt, int num_pages, cudaStream_t st);
// Shapes the tensor-core prefill kernel takes.
bool prefill_tc_supported(pa_dtype dt, int d, int dv, int group, int page_size);
cudaError_t launch_mla_tc(const AttnParams& p, pa_dtype dt, cudaStream_t st);
cudaError_t launch_backward(const void* q, const void* k, const void* v, const void* out, const float* lse,
                            const void* dout, float* dq, float* dk, float* dv, const SeqInfo* seqs, const int32_t* q2seq,
                            const int32_t* block_tables, int32_t table_width, int32_t page_size, int32_t hq,
                            int32_t hkv, int32_t d, int32_t dv_dim, float scale, int causal, int32_t window,
                            int64_t rows, pa_dtype dt, cudaStream_t st);
cudaError_t launch_mla_backward(const void* ql, const void* qr, const void* lat, const void* rope, const void* out,
                                const float* lse, const void* dout, float* dql, float* dqr, float* dlat, float* drope,
                                const SeqInfo* seqs, const int32_t* q2seq, const int32_t* block_tables,
                                int32_t table_width, int32_t page_size, int32_t h, int32_t r, int32_t pr, float scale,
                                int causal, int32_t window, int64_t rows, pa_dtype dt, cudaStream_t st);
cudaError_t launch_append(const void* new_k, const void* new_v, void* k_cache, void* v_cache, const SeqInfo* seqs,
                          const int32_t* q2seq, const int32_t* block_tables, int32_t table_width, int32_t page_size,
                          int32_t hkv, int32_t k_row_bytes, int32_t v_row_bytes, int64_t rows, cudaStream_t st);
// Tensor-core backward (backward_mma.cu): shapes it takes, its tile sizes and the launch of its
// three kernels (Drow, dK/dV, dQ).
bool backward_mma_supported(pa_dtype dt, int d, int dv, int group);
int backward_key_tile();
int backward_row_block();
// tcgen05 dK/dV kernel (backward_tc.cu): keys per CTA and launch; its 128-row blocks are read
// through TMA maps over Q and dO of num_queries rows.
int backward_tc_key_tile();
cudaError_t launch_backward_tc_dkdv(const BwdParams2& p, pa_dtype dt, int num_key_units, int64_t num_queries,
                                    cudaStream_t st);
// tcgen05 dQ kernel (backward_tc.cu): rows per CTA (128: 128 / G queries x G heads) and launch.
int backward_tc_row_block();
cudaError_t launch_backward_tc_dq(const BwdParams2& p, pa_dtype dt, int num_row_units, int64_t num_queries,
                                  cudaStream_t st);
cudaError_t launch_backward_mma(const BwdParams2& p, pa_dtype dt, int num_key_units, int num_row_units, int64_t rows,
                                int num_slot_sums, cudaStream_t st);
// Drow = dO . O per row (backward_mma.cu), for the other backward paths.
cudaError_t launch_bwd_dot(const void* out, const void* dout, float* drow, int64_t rows, int dv, pa_dtype dt,
                           cudaStream_t st);

// Tensor-core MLA backward (mla_backward_tc.cu): latent 512, rope 64, every sequence's rows
// (queries x heads) within one block of 128. Key tiles of 128 keys (two CTAs each: the latent's
// column halves), then dQ per (sequence, 64-column chunk of [latent | rope]).
struct MlaKeyTile {
    int32_t seq, k0, koff, pad;  // keys [k0, k0 + 128) of sequence seq; scratch key column koff + (t - k0)
};
struct MlaDqUnit {
    int32_t seq, k0, k1, koff;   // the sequence's key tiles cover [k0, k1); scratch columns from koff
};
struct MlaBwdTcParams {
    const void* ql;      // [Nq, H, 512]
    const void* qr;      // [Nq, H, 64]
    const void* lat;     // [P, ps, 1, 512]
    const void* rope;    // [P, ps, 1, 64]
    const void* dout;    // [Nq, H, 512]
    const float* lse;    // [Nq, H]
    const float* drow;   // [Nq, H] dO . O
    float* dql;          // [Nq, H, 512] written
    float* dqr;          // [Nq, H, 64] written
    float* dlat;         // [P, ps, 1, 512] added into
    float* drope;        // [P, ps, 1, 64] added into
    void* ds;            // [128][ds_cols] 16-bit scale * dS, row = the sequence's row (query x head)
    int64_t ds_cols;
    const SeqInfo* seqs;
    const int32_t* block_tables;
    const MlaKeyTile* tiles;
    const MlaDqUnit* dq_units;
    int32_t table_width, page_size, h, num_pages;
    float scale, scale_log2;
    int32_t causal, window;
    int* err;
};
constexpr int kMlaBwdKeyTile = 128;
bool mla_backward_tc_supported(pa_dtype dt, int latent_dim, int rope_dim, int num_heads);
cudaError_t launch_mla_backward_tc(const MlaBwdTcParams& p, pa_dtype dt, int num_tiles, int num_dq_units,
                                   int64_t num_queries, cudaStream_t st);
// Sparse top-K block selection (sparse.cu).
cudaError_t launch_sparse_scores(const void* q, const void* k, float* scores, int32_t sw, const SeqInfo* seqs,
                                 const int32_t* q2seq, const int32_t* block_tables, int32_t table_width,
                                 int32_t page_size, int32_t hq, int32_t hkv, int32_t d, int32_t block_size,
                                 float scale, int causal, int32_t window, int64_t num_queries, pa_dtype dt,
                                 cudaStream_t st);
cudaError_t launch_sparse_topk(const float* scores, int32_t sw, int32_t* sel, int32_t width, const SeqInfo* seqs,
                               const int32_t* q2seq, int32_t hkv, int32_t block_size, int32_t topk,
                               int32_t nb_max, int64_t num_queries, cudaStream_t st);
cudaError_t launch_sparse_prep(const int32_t* in, int32_t width, int32_t* out, int32_t wout, const SeqInfo* seqs,
                               const int32_t* q2seq, int32_t hkv, int32_t block_size, int32_t nb_max,
                               int64_t num_queries, int* err, cudaStream_t st);
// Shapes the tensor-core MLA decode kernel takes (one query per sequence).
bool mla_tc_supported(pa_dtype dt, int heads, int latent_dim, int rope_dim, int page_size);

// Largest row count (queries x group heads per KV head) the tensor-core decode kernel takes.
constexpr int kDecodeMaxRows = 16;

// Read-only facts of a plan, for entry points outside the plan's own translation unit.
struct PlanView {
    int device, num_sms;
    int32_t S, Nq, table_width, page_size, num_pages;
    const SeqInfo* host_seqs;
    const SeqInfo* d_seqs;
    const int32_t* d_bt;
    int* d_err;
};

// Validates a paged GQA call exactly as pa_forward does and fills `view`.
pa_status validated_gqa_view(pa_plan* P, const void* q, const void* k, const void* v, pa_dtype dtype, int32_t hq,
                             int32_t hkv, int32_t d, int32_t dv, float scale, int causal, int32_t window,
                             void* out, float* lse, PlanView* view);
// Thread-local error message of the C ABI (pa_last_error_message).
pa_status set_error(pa_status st, const char* fmt, ...);
pa_status clear_error();

// A non-blocking side stream of the library per device, with the two events of a fork/join: work
// that can run beside the caller's stream forks from it (an event recorded there) and joins back
// (an event recorded on the side stream that the caller's stream waits for), so a call stays
// stream-ordered and capturable. side_stream() is called with side_mutex() held, which also
// keeps each fork/join pair together.
struct SideStream {
    cudaStream_t stream = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr;
};
std::mutex& side_mutex();
cudaError_t side_stream(SideStream** out);

}  // namespace pa
