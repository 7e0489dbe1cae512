// C ABI of libfp2: argument validation, plan/workspace layout and dispatch.
//
// Everything here runs on the host.  No entry point allocates or frees
// device memory or synchronises, except fp2_status_check (which
// synchronises the stream and reads the 4-byte status word).
#include <algorithm>
#include <type_traits>
#include <cstring>
#include <mutex>
#include <vector>

#include <cuda.h>

#include "fp2_internal.h"

namespace fp2 {

namespace {

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct Carver {
    size_t off = 0;
    size_t take(size_t bytes) {
        size_t o = align_up(off, 256);
        off = o + bytes;
        return o;
    }
};

}  // namespace

int compute_layout(const fp2_problem* p, Layout* out) {
    if (!p || !out) return FP2_ERR_INVALID_ARG;
    if (p->num_seqs < 1 || !p->seqlens || !p->cu_seqlens) return FP2_ERR_INVALID_ARG;
    if (p->num_q_heads < 1 || p->num_kv_heads < 1) return FP2_ERR_INVALID_ARG;
    if (p->num_q_heads % p->num_kv_heads != 0) return FP2_ERR_INVALID_ARG;
    if (!(p->tau >= 0.0) || p->tau > 1e30) return FP2_ERR_INVALID_ARG;
    if (p->head_dim != 64 && p->head_dim != 128) return FP2_ERR_UNSUPPORTED;
    if (p->block_size != 64 && p->block_size != 128) return FP2_ERR_UNSUPPORTED;
    const int G = p->num_q_heads / p->num_kv_heads;
    if (G > kScoreQV) return FP2_ERR_UNSUPPORTED;
    if ((G * p->block_size) % kTileM != 0) return FP2_ERR_UNSUPPORTED;
    if (p->page_size != 0 && p->page_size != 64) return FP2_ERR_UNSUPPORTED;
    const bool chunked = p->q_seqlens != nullptr;
    if (chunked != (p->cu_q_seqlens != nullptr)) return FP2_ERR_INVALID_ARG;
    if ((p->prev_kbar != nullptr) != (p->prev_vbar != nullptr)) return FP2_ERR_INVALID_ARG;
    if (p->prev_kbar && (!chunked || (reinterpret_cast<uintptr_t>(p->prev_kbar) |
                                      reinterpret_cast<uintptr_t>(p->prev_vbar)) % 16 != 0))
        return FP2_ERR_INVALID_ARG;
    int64_t Tq = 0;
    if (chunked)
        for (int s = 0; s < p->num_seqs; ++s) {
            if (p->q_seqlens[s] < 1 || p->q_seqlens[s] > p->seqlens[s]) return FP2_ERR_INVALID_ARG;
            Tq += p->q_seqlens[s];
        }

    // a slice of a layer's heads, in place
    const int hkv_total = p->num_kv_heads_total ? p->num_kv_heads_total : p->num_kv_heads;
    if (p->kv_head_begin < 0 || p->num_kv_heads_total < 0 ||
        (int64_t)p->kv_head_begin + p->num_kv_heads > hkv_total)
        return FP2_ERR_INVALID_ARG;

    Dims d{};
    d.n_seqs = p->num_seqs;
    d.Hq = p->num_q_heads;
    d.Hkv = p->num_kv_heads;
    d.Hkv_str = hkv_total;
    d.Hq_str = G * hkv_total;
    d.head0 = p->kv_head_begin;
    d.G = G;
    d.d = p->head_dim;
    d.B = p->block_size;
    d.page_size = p->page_size;
    d.num_pages = p->num_pages;
    d.pt_stride = p->page_table_stride;
    d.tau = p->tau;
    d.rows_per_group = kScoreQV / G;

    int64_t T = 0, NB = 0, tri = 0, groups = 0, tiles = 0;
    int max_nb = 0, max_pages = 0;
    for (int s = 0; s < p->num_seqs; ++s) {
        const int64_t L = p->seqlens[s];
        if (L < 1 || L > (int64_t)1 << 30) return FP2_ERR_INVALID_ARG;
        const int64_t nb = (L + d.B - 1) / d.B;
        T += L;
        NB += nb;
        tri += nb * (nb + 1) / 2;
        groups += (nb + d.rows_per_group - 1) / d.rows_per_group;
        for (int64_t i0 = 0; i0 < nb; i0 += d.rows_per_group)
            tiles += (std::min<int64_t>(i0 + d.rows_per_group, nb) - 1) / kScoreKeys + 1;
        max_nb = std::max<int>(max_nb, (int)nb);
        max_pages = std::max<int>(max_pages, (int)((L + 63) / 64));
    }
    if (T > ((int64_t)1 << 31) - 1) return FP2_ERR_UNSUPPORTED;
    if (p->page_size == 64) {
        if (!p->page_table || p->num_pages < 1) return FP2_ERR_INVALID_ARG;
        if (p->page_table_stride < max_pages) return FP2_ERR_INVALID_ARG;
    }
    d.T = T;
    d.NB = NB;
    d.R = NB * d.Hkv;
    d.tri_total = tri;
    d.nnz_cap = tri * d.Hkv;
    if (d.nnz_cap > ((int64_t)1 << 31) - 1) return FP2_ERR_UNSUPPORTED;
    d.max_nb = max_nb;
    d.mask_words = (max_nb + 31) / 32;
    d.n_groups_cap = (int)groups;
    d.score_tiles = tiles;

    // attention schedule: split size from the layer's mean tiles per CTA,
    // then the work items and the split rows' slots
    SchedDims sd{};
    sd.n_mtiles = G * d.B / kTileM;
    sd.n_pairs = (sd.n_mtiles + 1) / 2;
    // rows of a chunked sequence start at the chunk's first query block
    auto first_row = [&](int s) -> int64_t {
        return chunked ? (int64_t)(p->seqlens[s] - p->q_seqlens[s]) / d.B : 0;
    };
    int64_t units = 0;
    for (int s = 0; s < p->num_seqs; ++s) {
        const int64_t nb = (p->seqlens[s] + d.B - 1) / d.B;
        for (int64_t i = first_row(s); i < nb; ++i) units += row_tile_bound(i, d.B);
    }
    // one attention CTA per SM of the current device (the attention kernel's grid)
    int64_t ctas = sm_count();
    if (ctas <= 0) ctas = kDefaultSchedSMs;
    const int64_t share = (units * d.Hkv * sd.n_pairs + ctas - 1) / ctas;
    const int64_t longest = row_tile_bound(max_nb - 1, d.B);
    int64_t split = std::max<int64_t>({(int64_t)kMinSplitTiles, (share + 1) / 2,
                                       (longest + kMaxSplits - 1) / kMaxSplits});
    // no splits when no item outlasts a CTA's mean share, or when the longest
    // row is too short to repay the merge
    if (longest <= share || longest < kMinSplitRow) split = 0;
    sd.split_c = (int)split;
    int64_t items = 0, slots = 0;
    for (int s = 0; s < p->num_seqs; ++s) {
        const int64_t nb = (p->seqlens[s] + d.B - 1) / d.B;
        for (int64_t i = first_row(s); i < nb; ++i) {
            const int S = row_splits(i, d.B, sd.split_c);
            items += S;
            if (S > 1) slots += S;
        }
    }
    sd.n_items = items * d.Hkv * sd.n_pairs;
    sd.split_slots = slots;
    if (sd.n_items > ((int64_t)1 << 31) - 1 || slots * d.Hkv > ((int64_t)1 << 31) - 1 ||
        row_splits(max_nb - 1, d.B, sd.split_c) > kMaxSplits || d.Hkv >= (1 << 16))
        return FP2_ERR_UNSUPPORTED;
    const int64_t head_kv_bytes = T * d.d * 4;   // bf16 K and V of one kv-head
    sd.heads_per_chunk = (int)std::max<int64_t>(1, std::min<int64_t>(d.Hkv, kSchedL2Bytes / head_kv_bytes));

    Layout& L = *out;
    std::memset(&L, 0, sizeof(L));
    L.dims = d;
    L.sched = sd;
    L.chunked = chunked;
    L.Tq = chunked ? Tq : T;
    fp2_plan_layout& pub = L.pub;
    pub.num_tokens = T;
    pub.num_blocks = NB;
    pub.num_rows = d.R;
    pub.nnz_cap = d.nnz_cap;
    pub.mask_words = d.mask_words;
    pub.max_blocks_per_seq = max_nb;

    const size_t n = (size_t)p->num_seqs;
    const size_t mean_elems = (size_t)NB * d.Hkv * d.d;
    Carver c;
    pub.off_status = c.take(sizeof(int32_t));
    L.off_meta_valid = c.take(sizeof(int32_t));
    pub.off_meta = L.off_meta_valid;
    pub.off_row_ptr = c.take(sizeof(int32_t) * (size_t)(d.R + 1));
    pub.off_col_idx = c.take(sizeof(int32_t) * (size_t)d.nnz_cap);
    pub.off_kept_mask = c.take(sizeof(uint32_t) * (size_t)d.R * d.mask_words);
    pub.off_kbar = c.take(sizeof(float) * mean_elems);
    pub.off_vbar = c.take(sizeof(float) * mean_elems);
    pub.off_kbar_bf16 = c.take(sizeof(uint16_t) * mean_elems);
    pub.off_vbar_bf16 = c.take(sizeof(uint16_t) * mean_elems);
    pub.off_kbar_e4m3 = c.take(mean_elems);
    pub.off_vbar_e4m3 = c.take(mean_elems);
    pub.off_kbar_e4m3_lo = c.take(mean_elems);
    pub.off_kbar_scale = c.take(sizeof(float) * (size_t)NB * d.Hkv);
    pub.off_vbar_scale = c.take(sizeof(float) * (size_t)NB * d.Hkv);
    L.off_cu_blocks = c.take(sizeof(int32_t) * (n + 1));
    L.off_block_seq = c.take(sizeof(int32_t) * (size_t)NB);
    L.off_tri_off = c.take(sizeof(int64_t) * (n + 1));
    L.off_group_cu = c.take(sizeof(int32_t) * (n + 1));
    L.off_group_seq = c.take(sizeof(int32_t) * (size_t)std::max<int64_t>(1, groups));
    L.off_tile_cu = c.take(sizeof(int32_t) * (size_t)(groups + 1));
    L.off_vmax = c.take(sizeof(float) * n * (size_t)d.Hkv);
    L.off_sched = c.take(sizeof(int4) * (size_t)sd.n_items);
    L.off_sched_cnt = c.take(sizeof(int32_t) * (size_t)max_nb);
    L.off_sched_off = c.take(sizeof(int64_t) * (size_t)max_nb);
    const size_t split_rows = (size_t)sd.split_slots * d.Hkv * d.G * d.B;
    L.off_split_o = c.take(sizeof(float) * split_rows * d.d);
    L.off_split_lse = c.take(sizeof(float) * split_rows);
    L.off_slot_item = c.take(sizeof(int32_t) * (size_t)sd.split_slots * d.Hkv);
    L.off_q_off = c.take(sizeof(int32_t) * n);
    L.off_thr_next = c.take(sizeof(int32_t));
    L.off_mean_amax = c.take(sizeof(uint32_t) * 2 * (size_t)NB * d.Hkv);
    L.off_csr_count = c.take(sizeof(int32_t) * (size_t)d.R);
    L.off_csr_seg = c.take(sizeof(int32_t) * (size_t)((d.R + kCsrRows - 1) / kCsrRows));
    L.off_csr_sup = c.take(sizeof(int32_t) * (size_t)((d.R + kCsrSup - 1) / kCsrSup));
    pub.plan_bytes = align_up(c.off, 256);

    Carver w;
    L.ws_qbar64 = w.take(sizeof(double) * (size_t)NB * d.Hq * d.d);
    L.ws_qbar32 = w.take(sizeof(float) * (size_t)NB * d.Hq * d.d);
    L.ws_kbar_tf = w.take(sizeof(float) * mean_elems);
    L.ws_kbar64 = w.take(sizeof(double) * mean_elems);
    L.ws_qnorm = w.take(sizeof(float) * (size_t)NB * d.Hkv);
    L.ws_qres = w.take(sizeof(float) * (size_t)NB * d.Hkv);
    L.ws_kb2 = w.take(sizeof(float2) * (size_t)NB * d.Hkv);
    L.ws_scores = w.take(sizeof(float) * (size_t)d.nnz_cap);
    L.ws_bounds = w.take(sizeof(double) * 2 * (size_t)d.R);
    pub.workspace_bytes = align_up(w.off, 256);
    pub.num_work_items = sd.n_items;
    pub.num_split_slots = sd.split_slots * d.Hkv;
    return FP2_OK;
}

PlanPtrs plan_ptrs(const Layout& L, void* plan) {
    char* b = static_cast<char*>(plan);
    const fp2_plan_layout& u = L.pub;
    PlanPtrs p;
    p.row_ptr = reinterpret_cast<int32_t*>(b + u.off_row_ptr);
    p.col_idx = reinterpret_cast<int32_t*>(b + u.off_col_idx);
    p.kept_mask = reinterpret_cast<uint32_t*>(b + u.off_kept_mask);
    p.kbar = reinterpret_cast<float*>(b + u.off_kbar);
    p.vbar = reinterpret_cast<float*>(b + u.off_vbar);
    p.kbar16 = reinterpret_cast<uint16_t*>(b + u.off_kbar_bf16);
    p.vbar16 = reinterpret_cast<uint16_t*>(b + u.off_vbar_bf16);
    p.kbar8 = reinterpret_cast<uint8_t*>(b + u.off_kbar_e4m3);
    p.kbar8lo = reinterpret_cast<uint8_t*>(b + u.off_kbar_e4m3_lo);
    p.vbar8 = reinterpret_cast<uint8_t*>(b + u.off_vbar_e4m3);
    p.kbar_scale = reinterpret_cast<float*>(b + u.off_kbar_scale);
    p.vbar_scale = reinterpret_cast<float*>(b + u.off_vbar_scale);
    p.status = reinterpret_cast<int32_t*>(b + u.off_status);
    p.meta_valid = reinterpret_cast<int32_t*>(b + L.off_meta_valid);
    p.cu_blocks = reinterpret_cast<int32_t*>(b + L.off_cu_blocks);
    p.block_seq = reinterpret_cast<int32_t*>(b + L.off_block_seq);
    p.tri_off = reinterpret_cast<int64_t*>(b + L.off_tri_off);
    p.group_cu = reinterpret_cast<int32_t*>(b + L.off_group_cu);
    p.group_seq = reinterpret_cast<int32_t*>(b + L.off_group_seq);
    p.tile_cu = reinterpret_cast<int32_t*>(b + L.off_tile_cu);
    p.vmax = reinterpret_cast<float*>(b + L.off_vmax);
    p.sched = reinterpret_cast<int4*>(b + L.off_sched);
    p.sched_cnt = reinterpret_cast<int32_t*>(b + L.off_sched_cnt);
    p.sched_off = reinterpret_cast<int64_t*>(b + L.off_sched_off);
    p.split_o = reinterpret_cast<float*>(b + L.off_split_o);
    p.split_lse = reinterpret_cast<float*>(b + L.off_split_lse);
    p.slot_item = reinterpret_cast<int32_t*>(b + L.off_slot_item);
    p.q_off = reinterpret_cast<int32_t*>(b + L.off_q_off);
    p.thr_next = reinterpret_cast<int32_t*>(b + L.off_thr_next);
    p.mean_amax = reinterpret_cast<uint32_t*>(b + L.off_mean_amax);
    p.csr_count = reinterpret_cast<int32_t*>(b + L.off_csr_count);
    p.csr_seg = reinterpret_cast<int32_t*>(b + L.off_csr_seg);
    p.csr_sup = reinterpret_cast<int32_t*>(b + L.off_csr_sup);
    p.cu_q = nullptr;
    return p;
}

WsPtrs ws_ptrs(const Layout& L, void* ws) {
    char* b = static_cast<char*>(ws);
    WsPtrs w;
    w.qbar64 = reinterpret_cast<double*>(b + L.ws_qbar64);
    w.qbar32 = reinterpret_cast<float*>(b + L.ws_qbar32);
    w.kbar_tf = reinterpret_cast<float*>(b + L.ws_kbar_tf);
    w.kbar64 = reinterpret_cast<double*>(b + L.ws_kbar64);
    w.qnorm = reinterpret_cast<float*>(b + L.ws_qnorm);
    w.qres = reinterpret_cast<float*>(b + L.ws_qres);
    w.kb2 = reinterpret_cast<float2*>(b + L.ws_kb2);
    w.scores = reinterpret_cast<float*>(b + L.ws_scores);
    w.bounds = reinterpret_cast<double*>(b + L.ws_bounds);
    return w;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// against the driver library).
static EncodeTiledFn get_encode() {
    static std::once_flag once;
    static EncodeTiledFn fn = nullptr;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

bool make_tensor_map(void* map, const void* base, int rank, const uint64_t* dims,
                     const uint64_t* strides, const uint32_t* box, MapType type) {
    EncodeTiledFn enc = get_encode();
    if (!enc) return false;
    const cuuint32_t elem_strides[5] = {1, 1, 1, 1, 1};
    const CUtensorMapDataType dt = type == kMapF32  ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                   : type == kMapU8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                                    : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const CUresult r = enc(static_cast<CUtensorMap*>(map), dt, static_cast<cuuint32_t>(rank),
                           const_cast<void*>(base), reinterpret_cast<const cuuint64_t*>(dims),
                           reinterpret_cast<const cuuint64_t*>(strides),
                           reinterpret_cast<const cuuint32_t*>(box), elem_strides,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

int sm_count() {
    static std::mutex mu;
    static std::vector<int> cache;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();   // no device visible: leave no sticky error behind
        return 0;
    }
    std::lock_guard<std::mutex> lock(mu);
    if ((int)cache.size() <= dev) cache.resize(dev + 1, 0);
    if (cache[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
        cache[dev] = n;
    }
    return cache[dev];
}

}  // namespace fp2

using namespace fp2;

namespace {

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// The first element of a head slice: `heads` heads of `elt`-byte elements
// past the tensor's start (the tensors keep all heads of each token).
template <typename T>
T* head_offset(T* p, int64_t heads, int d, int elt) {
    if (!p) return p;
    using B = typename std::conditional<std::is_const<T>::value, const char, char>::type;
    return reinterpret_cast<T*>(reinterpret_cast<B*>(p) + heads * d * elt);
}

}  // namespace

extern "C" {

int fp2_version(void) { return FP2_VERSION; }

const char* fp2_strerror(int code) {
    switch (code) {
        case FP2_OK: return "ok";
        case FP2_ERR_INVALID_ARG: return "invalid argument";
        case FP2_ERR_UNSUPPORTED: return "unsupported configuration";
        case FP2_ERR_CAPACITY: return "caller buffer too small";
        case FP2_ERR_CUDA: return "CUDA error";
        case FP2_ERR_TIMEOUT: return "device-side wait timed out";
        case FP2_ERR_DEVICE_CHECK: return "device-side consistency check failed";
        default: return "unknown error";
    }
}

int fp2_plan_sizes(const fp2_problem* problem, fp2_plan_layout* layout) {
    if (!layout) return FP2_ERR_INVALID_ARG;
    Layout L;
    int rc = compute_layout(problem, &L);
    if (rc != FP2_OK) return rc;
    *layout = L.pub;
    return FP2_OK;
}

int fp2_plan(const fp2_problem* problem, const void* q, const void* k, const void* v, void* plan,
             size_t plan_bytes, void* workspace, size_t workspace_bytes, void* stream) {
    Layout L;
    int rc = compute_layout(problem, &L);
    if (rc != FP2_OK) return rc;
    if (!q || !k || !v || !plan || !workspace) return FP2_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16)) return FP2_ERR_INVALID_ARG;
    if (!aligned(plan, 256) || !aligned(workspace, 256)) return FP2_ERR_INVALID_ARG;
    if (plan_bytes < L.pub.plan_bytes || workspace_bytes < L.pub.workspace_bytes)
        return FP2_ERR_CAPACITY;
    const Dims& D = L.dims;
    return launch_plan(L, problem, head_offset(q, (int64_t)D.G * D.head0, D.d, 2),
                       head_offset(k, D.head0, D.d, 2), head_offset(v, D.head0, D.d, 2),
                       plan_ptrs(L, plan), ws_ptrs(L, workspace), static_cast<cudaStream_t>(stream));
}

int fp2_plan_kv8(const fp2_problem* problem, const void* q, const void* k_e4m3, const void* v_e4m3,
                 const float* k_scale, const float* v_scale, void* plan, size_t plan_bytes,
                 void* workspace, size_t workspace_bytes, void* stream) {
    Layout L;
    int rc = compute_layout(problem, &L);
    if (rc != FP2_OK) return rc;
    if (L.chunked) return FP2_ERR_UNSUPPORTED;   // chunks over an FP8 cache: not built
    if (!q || !k_e4m3 || !v_e4m3 || !k_scale || !v_scale || !plan || !workspace)
        return FP2_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k_e4m3, 16) || !aligned(v_e4m3, 16) || !aligned(k_scale, 4) ||
        !aligned(v_scale, 4) || !aligned(plan, 256) || !aligned(workspace, 256))
        return FP2_ERR_INVALID_ARG;
    if (plan_bytes < L.pub.plan_bytes || workspace_bytes < L.pub.workspace_bytes)
        return FP2_ERR_CAPACITY;
    const Dims& D = L.dims;
    return launch_plan(L, problem, head_offset(q, (int64_t)D.G * D.head0, D.d, 2),
                       head_offset(k_e4m3, D.head0, D.d, 1), head_offset(v_e4m3, D.head0, D.d, 1),
                       plan_ptrs(L, plan), ws_ptrs(L, workspace), static_cast<cudaStream_t>(stream),
                       k_scale, v_scale);
}

int fp2_quantize_fp8(const fp2_problem* problem, const void* plan, size_t plan_bytes, const void* x,
                     int32_t which, void* x_e4m3, float* scales, void* stream) {
    Layout L;
    int rc = compute_layout(problem, &L);
    if (rc != FP2_OK) return rc;
    if (!plan || !x || !x_e4m3 || !scales || which < 0 || which > 2) return FP2_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(x_e4m3, 16) || !aligned(scales, 4) || !aligned(plan, 256))
        return FP2_ERR_INVALID_ARG;
    if (plan_bytes < L.pub.plan_bytes) return FP2_ERR_CAPACITY;
    const Dims& D = L.dims;
    const int64_t h0 = which == 0 ? (int64_t)D.G * D.head0 : D.head0;
    const void* xs[1] = {head_offset(x, h0, D.d, 2)};
    void* x8s[1] = {head_offset(x_e4m3, h0, D.d, 1)};
    float* ss[1] = {scales};
    return launch_quantize(L, problem, plan_ptrs(L, const_cast<void*>(plan)), xs, x8s, ss, which, 1,
                           static_cast<cudaStream_t>(stream));
}

int fp2_quantize_fp8_qkv(const fp2_problem* problem, const void* plan, size_t plan_bytes,
                         const void* q, const void* k, const void* v, void* q_e4m3, void* k_e4m3,
                         void* v_e4m3, float* q_scales, float* k_scales, float* v_scales,
                         void* stream) {
    Layout L;
    int rc = compute_layout(problem, &L);
    if (rc != FP2_OK) return rc;
    const void* xs[3] = {q, k, v};
    void* x8s[3] = {q_e4m3, k_e4m3, v_e4m3};
    float* ss[3] = {q_scales, k_scales, v_scales};
    if (!plan || !aligned(plan, 256)) return FP2_ERR_INVALID_ARG;
    for (int w = 0; w < 3; ++w)
        if (!xs[w] || !x8s[w] || !ss[w] || !aligned(xs[w], 16) || !aligned(x8s[w], 16) ||
            !aligned(ss[w], 4))
            return FP2_ERR_INVALID_ARG;
    if (plan_bytes < L.pub.plan_bytes) return FP2_ERR_CAPACITY;
    const Dims& D = L.dims;
    const int64_t hq0 = (int64_t)D.G * D.head0;
    xs[0] = head_offset(q, hq0, D.d, 2);
    xs[1] = head_offset(k, D.head0, D.d, 2);
    xs[2] = head_offset(v, D.head0, D.d, 2);
    x8s[0] = head_offset(q_e4m3, hq0, D.d, 1);
    x8s[1] = head_offset(k_e4m3, D.head0, D.d, 1);
    x8s[2] = head_offset(v_e4m3, D.head0, D.d, 1);
    return launch_quantize(L, problem, plan_ptrs(L, const_cast<void*>(plan)), xs, x8s, ss, 0, 3,
                           static_cast<cudaStream_t>(stream));
}

int fp2_prefill(const fp2_problem* problem, const void* plan, size_t plan_bytes, const void* q,
                const void* k, const void* v, const float* q_scale, const float* k_scale,
                const float* v_scale, int32_t dtype, void* o, float* lse, uint32_t flags,
                void* stream) {
    Layout L;
    int rc = compute_layout(problem, &L);
    if (rc != FP2_OK) return rc;
    if (!plan || !q || !k || !v || !o || !lse) return FP2_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
        !aligned(lse, 4) || !aligned(plan, 256))
        return FP2_ERR_INVALID_ARG;
    if (plan_bytes < L.pub.plan_bytes) return FP2_ERR_CAPACITY;
    if (dtype == FP2_DTYPE_BF16) {
        if (q_scale || k_scale || v_scale) return FP2_ERR_INVALID_ARG;
    } else if (dtype == FP2_DTYPE_E4M3) {
        if (!q_scale || !k_scale || !v_scale) return FP2_ERR_INVALID_ARG;
        if (!aligned(q_scale, 4) || !aligned(k_scale, 4) || !aligned(v_scale, 4))
            return FP2_ERR_INVALID_ARG;
        if (L.dims.d != 128) return FP2_ERR_UNSUPPORTED;
    } else {
        return FP2_ERR_INVALID_ARG;
    }
    const uint32_t known = FP2_NO_CORRECTION | FP2_DEBUG_DROP_Q_LOAD;
    if (flags & ~known) return FP2_ERR_INVALID_ARG;
    const Dims& D = L.dims;
    const int elt = dtype == FP2_DTYPE_E4M3 ? 1 : 2;
    const int64_t hq0 = (int64_t)D.G * D.head0;
    // lse is [G * num_kv_heads_total, Tq]: the slice's rows are contiguous
    return launch_prefill(L, problem, plan_ptrs(L, const_cast<void*>(plan)),
                          head_offset(q, hq0, D.d, elt), head_offset(k, D.head0, D.d, elt),
                          head_offset(v, D.head0, D.d, elt), q_scale, k_scale, v_scale, dtype,
                          head_offset(o, hq0, D.d, 2), lse + hq0 * L.Tq, flags,
                          static_cast<cudaStream_t>(stream));
}

int fp2_status_check(const void* plan, size_t plan_bytes, void* stream, int32_t* device_status) {
    if (!plan || plan_bytes < 4) return FP2_ERR_INVALID_ARG;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return FP2_ERR_CUDA;
    int32_t st = 0;
    // The status word is the first field of the plan buffer (offset 0).
    if (cudaMemcpy(&st, plan, sizeof(st), cudaMemcpyDeviceToHost) != cudaSuccess) return FP2_ERR_CUDA;
    if (device_status) *device_status = st;
    if (st == 0) return FP2_OK;
    if (st & FP2_STATUS_TIMEOUT) return FP2_ERR_TIMEOUT;
    return FP2_ERR_DEVICE_CHECK;
}

}  // extern "C"
