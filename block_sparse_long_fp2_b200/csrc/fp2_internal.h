// Internal declarations shared by the libfp2 translation units.
//
// Layout of the plan buffer and of fp2_plan's workspace, the derived
// problem sizes every kernel needs, and the kernel launchers.
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda_runtime.h>

#include "fp2.h"

namespace fp2 {

// Query rows of one PackGQA tile (M of one tcgen05 MMA).
constexpr int kTileM = 128;
// CSR rows per CTA of the threshold kernel (one warp per row).
constexpr int kThrRows = 8;    // threshold: warps (rows in flight) per CTA
constexpr int kCsrRows = 32;     // CSR offsets: rows per segment
constexpr int kCsrSup = 1024;    // rows per super-segment (kCsrRows segments)
// Query vectors scored together by one CTA of the scoring kernel (MMA M).
constexpr int kScoreQV = 128;
// Key blocks scored together by one CTA of the scoring kernel (MMA N).
constexpr int kScoreKeys = 128;

// Attention work schedule.  The rows of one chunk of kv-heads are taken
// longest first; a chunk holds as many kv-heads as keep their bf16 K and V
// within kSchedL2Bytes, so the CTAs that run together share K/V in L2.  When
// the longest row's tile bound exceeds a CTA's mean share of the layer (taken
// over one CTA per SM of the current device, kDefaultSchedSMs when no device
// is visible) and kMinSplitRow tiles, every row whose bound exceeds
// half that share is cut into count-balanced splits of at least
// kMinSplitTiles tiles (at most kMaxSplits), merged afterwards by their
// log-sum-exp.  (The merge costs a launch of about 10 us; on a 16-row layer
// with 17-tile rows, splitting measured slower than not.)
constexpr int64_t kSchedL2Bytes = (int64_t)64 << 20;
constexpr int kDefaultSchedSMs = 148;   // a B200
constexpr int kMinSplitTiles = 8;
constexpr int kMinSplitRow = 32;
constexpr int kMaxSplits = 32;   // splits of one row (the merge takes one per lane)
// Passes over the grid up to which CTAs alternate their direction through the
// schedule (fewer, longer items per CTA: evens out the decreasing lengths).
constexpr int kZigZagMaxPasses = 16;

// Upper bound of the tiles of row i (kept blocks 0..i plus pseudo tiles of
// B block means each) and the number of splits it gets for split size c
// (0: rows are never split).
__host__ __device__ inline int64_t row_tile_bound(int64_t i, int B) { return i + 1 + (i + B - 1) / B; }
__host__ __device__ inline int row_splits(int64_t i, int B, int c) {
    return c ? (int)((row_tile_bound(i, B) + c - 1) / c) : 1;
}

// Derived sizes of one problem (host computed, passed to kernels by value).
struct Dims {
    int n_seqs;
    int Hq, Hkv, G, d, B;
    int Hq_str, Hkv_str;  // heads per token of the q / o and k / v tensors (>= Hq, Hkv for a slice)
    int head0;            // first kv-head of the slice in those tensors
    int page_size, num_pages, pt_stride;
    int mask_words;       // 32-bit words per kept-mask row
    int max_nb;           // largest nb_s
    int rows_per_group;   // query blocks per scoring CTA (kScoreQV / G)
    int n_groups_cap;     // upper bound of scoring row groups per kv-head
    int64_t T, NB, R, tri_total, nnz_cap;
    int64_t score_tiles;  // (query group, 128-key-block chunk) tiles inside the causal triangles
    double tau;
};

// Sizes of the attention schedule (host computed; passed only to the kernels
// that build or read the schedule).
struct SchedDims {
    int n_mtiles;           // 128-row query tiles per row, G * B / 128
    int n_pairs;            // work items per row split, ceil(n_mtiles / 2)
    int split_c;            // split size in tiles (0: no row is split)
    int heads_per_chunk;    // kv-heads per schedule chunk
    int64_t n_items;        // work items of the layer
    int64_t split_slots;    // row splits of split rows, per kv-head
};

// Block and token offsets of up to kMapSeqs sequences, computed on the host
// from the problem's host arrays and passed to the pooling kernel by value,
// so that it needs no device-side map and can run before k_meta.
constexpr int kMapSeqs = 64;
struct SeqMap {
    int32_t n;
    int32_t cu_blocks[kMapSeqs + 1];
    int32_t cu_tok[kMapSeqs + 1];
    int32_t cu_q[kMapSeqs + 1];   // query tokens (chunked prefill), else cu_tok
    int32_t q_off[kMapSeqs];      // position of the first query (L - Q, else 0)
};

// Device pointers into the plan buffer.
struct PlanPtrs {
    int32_t* row_ptr;
    int32_t* col_idx;
    uint32_t* kept_mask;
    float* kbar;
    float* vbar;
    uint16_t* kbar16;
    uint16_t* vbar16;
    uint8_t* kbar8;
    uint8_t* kbar8lo;   // e4m3 residual of kbar / chunk scale - kbar8
    uint8_t* vbar8;
    float* kbar_scale;
    float* vbar_scale;
    int32_t* status;
    // private meta
    int32_t* meta_valid;   // [1]  1 when cu_seqlens passed the device checks
    int32_t* cu_blocks;    // [n+1]
    int32_t* block_seq;    // [NB]
    int64_t* tri_off;      // [n+1] prefix of nb (nb + 1) / 2
    int32_t* group_cu;     // [n+1] prefix of scoring CTAs per sequence
    int32_t* group_seq;    // [n_groups_cap]
    int32_t* tile_cu;      // [n_groups_cap+1] prefix of scoring tiles per row group
    float* vmax;           // [n, Hkv]  largest V scale of each sequence and kv-head (FP8)
    int4* sched;           // [n_items]  {global block, g | pair << 16, split | splits << 16, slot}
    int32_t* sched_cnt;    // [max_nb]   sequences longer than i blocks
    int64_t* sched_off;    // [max_nb]   items of one kv-head's rows with a larger i
    float* split_o;        // [Hkv * split_slots, G * B, d]  O of one split (normalised)
    float* split_lse;      // [Hkv * split_slots, G * B]     its log2-sum-exp
    int32_t* slot_item;    // [Hkv * split_slots]  schedule index of the slot's row (split 0, pair 0)
    int32_t* q_off;        // [n]  position of the first query (L - Q for a chunk, else 0)
    // the threshold kernel's single-pass CSR prefix sum (decoupled look-back):
    // a CTA ticket counter and one flag word per CTA, zeroed by k_meta
    int32_t* thr_next;     // [1]: the threshold's next item
    uint32_t* mean_amax;   // [NB, Hkv, 2]: absmax of the K / V means of the chunk starting at the block
    int32_t* csr_count;    // [R]: kept blocks per row
    int32_t* csr_seg;      // [ceil(R / kCsrRows)]: kept blocks per segment of kCsrRows rows
    int32_t* csr_sup;      // [ceil(R / kCsrSup)]: kept blocks per super-segment of kCsrSup rows
    const int32_t* cu_q;   // caller's cu_q_seqlens for a chunked problem, else null (set per call)
};

// Device pointers into fp2_plan's workspace.
struct WsPtrs {
    double* qbar64;   // [NB, Hq, d]
    float* qbar32;    // [NB, Hq, d]  the same means rounded to tf32 (stored as fp32)
    float* kbar_tf;   // [NB, Hkv, d] the key means rounded to tf32 (stored as fp32)
    double* kbar64;   // [NB, Hkv, d]
    float* qnorm;     // [NB, Hkv]  max over the group's heads of |Qbar|_2 (rounded up)
    float* qres;      // [NB, Hkv]  max over the group's heads of |Qbar - tf32(Qbar)|_2 (rounded up)
    float2* kb2;      // [Hkv, NB]  (|Kbar|_2, |Kbar - tf32(Kbar)|_2 + c_d (|Kbar|_2 + that)),
                      //   both rounded up, contiguous over a head's blocks
    float* scores;    // [Hkv, tri_total] fp32 block scores, row (s,g,i) at
                      //   g * tri_total + tri_off[s] + i (i + 1) / 2 + j
    double* bounds;   // [R, 2] per row: the largest lower and upper bound of any
                      //   score (sc_j -/+ its error bound), from the pipelined scorer
};

struct Layout {
    Dims dims;
    SchedDims sched;
    bool chunked;   // q holds a chunk of each sequence (q_seqlens given)
    int64_t Tq;     // query tokens (T unless chunked)
    fp2_plan_layout pub;
    size_t off_meta_valid, off_cu_blocks, off_block_seq, off_tri_off, off_group_cu, off_group_seq,
        off_tile_cu, off_vmax, off_sched, off_sched_cnt, off_sched_off, off_split_o, off_split_lse,
        off_slot_item, off_q_off, off_thr_next, off_mean_amax, off_csr_count, off_csr_seg, off_csr_sup;
    size_t ws_qbar64, ws_qbar32, ws_kbar_tf, ws_kbar64, ws_qnorm, ws_qres, ws_kb2, ws_scores,
        ws_bounds;
};

// Validates the problem on the host and computes sizes and offsets.
int compute_layout(const fp2_problem* p, Layout* out);
PlanPtrs plan_ptrs(const Layout& L, void* plan);
WsPtrs ws_ptrs(const Layout& L, void* ws);

// Launchers (return FP2_OK or FP2_ERR_CUDA).
// k_scale / v_scale non-null: k and v are e4m3 codes with per-(block, kv-head)
// scales (planning from an FP8 KV cache); otherwise bf16.
int launch_plan(const Layout& L, const fp2_problem* p, const void* q, const void* k,
                const void* v, const PlanPtrs& pp, const WsPtrs& ws, cudaStream_t st,
                const float* k_scale = nullptr, const float* v_scale = nullptr);
// Quantises count tensors (which = first .. first + count - 1: 0 q, 1 k, 2 v)
// in one launch.
int launch_quantize(const Layout& L, const fp2_problem* p, const PlanPtrs& pp, const void* const* x,
                    void* const* x8, float* const* scales, int first, int count, cudaStream_t st);
int launch_prefill(const Layout& L, const fp2_problem* p, const PlanPtrs& pp, const void* q,
                   const void* k, const void* v, const float* qs, const float* ks,
                   const float* vs, int dtype, void* o, float* lse, uint32_t flags,
                   cudaStream_t st);

// Number of SMs of the current device (cached per device).
int sm_count();

// A tiled TMA tensor map with 128-byte swizzle over `rank` dimensions
// (innermost first; strides in bytes for dimensions 1..rank-1).  Element
// types: bf16, uint8 (e4m3 codes) and fp32.  False when the driver rejects it.
enum MapType { kMapBF16 = 0, kMapU8 = 1, kMapF32 = 2 };
bool make_tensor_map(void* map, const void* base, int rank, const uint64_t* dims,
                     const uint64_t* strides, const uint32_t* box, MapType type);

}  // namespace fp2
