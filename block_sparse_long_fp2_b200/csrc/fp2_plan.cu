// Stage 1 of FlashPrefill V2 ("pattern discovery", Figure 3 of the
// metallab.ai summary of arXiv 2608.19758): block-mean pooling, block
// scores under PackGQA, max-based thresholding and the CSR block index.
//
// Kernels, in launch order:
//   pool     HBM-bound: streams Q, K, V once with 16-byte coalesced loads and
//            accumulates each block's sum in float64 (exact for bf16 inputs),
//            writing Qbar (fp64 workspace) and Kbar/Vbar (fp32, bf16, fp64),
//            and the norms |Qbar|, |Kbar| of the score error bound.  For up to
//            64 sequences it takes the block map by value and runs first.
//   meta     one CTA, a programmatic dependent of the pool (it runs beside the
//            pool's last wave): checks cu_seqlens (and a chunk's
//            cu_q_seqlens), derives block / scoring-group maps, the chunk
//            offsets and the attention kernel's work schedule.
//   (norms   |Qbar|, |Kbar| when the pool cannot: G query heads of a kv-head
//            not within one pooling CTA.)
//   score    persistent, one CTA per SM: tf32 tcgen05 MMAs
//            of the means rounded to tf32 (exact products, fp32 sums), max over
//            the group's heads, to a scratch array; also each row's bounds of
//            its largest score.
//   threshold  one warp per row, rows taken longest first: the threshold
//            decision.  A block whose score lies within the scores' error
//            bound of the threshold, and an undecided row's candidates for
//            its maximum, are re-scored in float64, so the kept set is the one
//            float64 scores give.  Before the rows, its warps take the
//            absolute maxima of the e4m3 block means' chunks (one scale per
//            chunk of B blocks, a pseudo tile of the FP8 correction).
//   csr      the CSR row pointers (each warp adds up the kept counts of
//            the rows before its row, by segments), then the column ids;
//            before the rows, the e4m3 codes of the block means.
#include <cfloat>
#include <cstring>
#include <cmath>

#include "fp2_device.cuh"

namespace fp2 {

namespace {

// ---------------------------------------------------------------------------
// meta: sequence -> block and scoring-group maps, device-side checks, and the
// attention kernel's work schedule
// ---------------------------------------------------------------------------

constexpr int kMetaThreads = 1024;

// Exclusive prefix sum of v over the CTA (blockDim.x == kMetaThreads); every
// thread gets the CTA's total in *total.
__device__ int64_t block_excl_scan(int64_t v, int64_t* total) {
    __shared__ int64_t warp_sum[kMetaThreads / 32];
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    int64_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int64_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) warp_sum[w] = x;
    __syncthreads();
    if (w == 0) {
        int64_t t = warp_sum[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int64_t y = __shfl_up_sync(0xffffffffu, t, o);
            if (lane >= o) t += y;
        }
        warp_sum[lane] = t;
    }
    __syncthreads();
    const int64_t before = (w ? warp_sum[w - 1] : 0) + x - v;
    *total = warp_sum[kMetaThreads / 32 - 1];
    __syncthreads();
    return before;
}

// Whether sequence s has a row for query block i: i below its block count and
// not below the first query block of its chunk.
__device__ __forceinline__ bool has_row(const Dims& D, const PlanPtrs& P, int s, int i) {
    return i < P.cu_blocks[s + 1] - P.cu_blocks[s] && i >= P.q_off[s] / D.B;
}

// The attention kernel's work items in the order its CTAs take them: kv-head
// chunks in order; inside a chunk the rows by block index i, largest first,
// then kv-head, then sequence; inside a row its splits, then its query-tile
// pairs.  Rows with the same i have the same number of items, so every
// row's position follows from prefix sums over i.
__device__ void build_schedule(const Dims& D, const SchedDims& S, const PlanPtrs& P) {
    for (int i = threadIdx.x; i < D.max_nb; i += blockDim.x) {
        int c = 0;
        for (int s = 0; s < D.n_seqs; ++s) c += has_row(D, P, s, i) ? 1 : 0;
        P.sched_cnt[i] = c;
    }
    __syncthreads();
    // sched_off[i]: items of one kv-head's rows with a larger i (suffix sums,
    // blockDim.x entries at a time from the largest i down)
    int64_t per_head = 0, slots = 0;
    for (int base = 0; base < D.max_nb; base += blockDim.x) {
        const int i = D.max_nb - 1 - (base + (int)threadIdx.x);
        int64_t v = 0, sv = 0;
        if (i >= 0) {
            const int ns = row_splits(i, D.B, S.split_c);
            v = (int64_t)P.sched_cnt[i] * ns * S.n_pairs;
            sv = ns > 1 ? (int64_t)P.sched_cnt[i] * ns : 0;
        }
        int64_t tot, stot;
        const int64_t ex = block_excl_scan(v, &tot);
        block_excl_scan(sv, &stot);
        if (i >= 0) P.sched_off[i] = per_head + ex;
        per_head += tot;
        slots += stot;
    }
    if (per_head * D.Hkv != S.n_items || slots != S.split_slots) {
        if (threadIdx.x == 0) {
            *P.meta_valid = 0;
            atomicOr(P.status, (int32_t)FP2_STATUS_BAD_SEQLENS);
        }
        return;
    }
    __syncthreads();
    for (int64_t b = threadIdx.x; b < D.NB; b += blockDim.x) {
        const int s = P.block_seq[b];
        const int i = (int)(b - P.cu_blocks[s]);
        if (!has_row(D, P, s, i)) continue;   // query block below the chunk
        int rank = 0;   // earlier sequences that also have a row i
        for (int s2 = 0; s2 < s; ++s2) rank += has_row(D, P, s2, i) ? 1 : 0;
        const int ns = row_splits(i, D.B, S.split_c);
        const int64_t w = (int64_t)ns * S.n_pairs;
        const int64_t cnt = P.sched_cnt[i], off = P.sched_off[i];
        for (int g = 0; g < D.Hkv; ++g) {
            const int g0 = g - g % S.heads_per_chunk;
            const int nh = min(S.heads_per_chunk, D.Hkv - g0);
            const int64_t in_chunk = off * nh + ((g - g0) * cnt + rank) * w;
            const int64_t first = (int64_t)g0 * per_head + in_chunk;
            // split rows come first in their chunk, so their items, counted in
            // row splits, number the split slots
            const int slot = ns > 1 ? (int)((int64_t)g0 * S.split_slots + in_chunk / S.n_pairs) : 0;
            if (ns > 1)
                for (int k = 0; k < ns; ++k) P.slot_item[slot + k] = (int32_t)first;
            for (int k = 0; k < ns; ++k)
                for (int mp = 0; mp < S.n_pairs; ++mp)
                    P.sched[first + (int64_t)k * S.n_pairs + mp] =
                        make_int4((int)b, g | (mp << 16), k | (ns << 16), slot);
        }
    }
}

__device__ void meta_maps(const Dims& D, const SchedDims& S, const int32_t* __restrict__ cu_seqlens,
                          const int32_t* __restrict__ page_table, const PlanPtrs& P);

// P.cu_q: prefix sums of a chunk's query counts (chunked prefill), or null;
// Tq their total.
__global__ void __launch_bounds__(kMetaThreads, 1) k_meta(Dims D, SchedDims S, const int32_t* __restrict__ cu_seqlens,
                       const int32_t* __restrict__ page_table, int64_t Tq, PlanPtrs P) {
    // the next kernel may be launched early: it waits for this one first
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int32_t* __restrict__ cu_q = P.cu_q;
    __shared__ int s_valid;
    if (threadIdx.x == 0) {
        int valid = cu_seqlens[0] == 0 && (!cu_q || cu_q[0] == 0);
        int64_t nb_sum = 0, tri = 0, grp = 0;
        for (int s = 0; s < D.n_seqs && valid; ++s) {
            const int64_t L = (int64_t)cu_seqlens[s + 1] - cu_seqlens[s];
            if (L < 1) { valid = 0; break; }
            const int64_t Q = cu_q ? (int64_t)cu_q[s + 1] - cu_q[s] : L;
            if (Q < 1 || Q > L) { valid = 0; break; }
            P.q_off[s] = (int32_t)(L - Q);
            const int64_t nb = (L + D.B - 1) / D.B;
            if (nb > D.max_nb) { valid = 0; break; }
            if (D.page_size && (L + 63) / 64 > D.pt_stride) { valid = 0; break; }
            P.cu_blocks[s] = (int32_t)nb_sum;
            P.tri_off[s] = tri;
            P.group_cu[s] = (int32_t)grp;
            nb_sum += nb;
            tri += nb * (nb + 1) / 2;
            grp += (nb + D.rows_per_group - 1) / D.rows_per_group;
            if (nb_sum > D.NB || grp > D.n_groups_cap) { valid = 0; break; }
        }
        if (valid) {
            valid = (cu_seqlens[D.n_seqs] == D.T) && (nb_sum == D.NB) && (tri == D.tri_total) &&
                    (!cu_q || cu_q[D.n_seqs] == Tq);
            P.cu_blocks[D.n_seqs] = (int32_t)nb_sum;
            P.tri_off[D.n_seqs] = tri;
            P.group_cu[D.n_seqs] = (int32_t)grp;
            // scoring tiles per row group: the 128-key-block chunks its rows reach
            int64_t tiles = 0;
            for (int s = 0; s < D.n_seqs; ++s) {
                const int nb = P.cu_blocks[s + 1] - P.cu_blocks[s];
                for (int gi = P.group_cu[s], i0 = 0; gi < P.group_cu[s + 1]; ++gi, i0 += D.rows_per_group) {
                    P.tile_cu[gi] = (int32_t)tiles;
                    tiles += (min(i0 + D.rows_per_group, nb) - 1) / kScoreKeys + 1;
                }
            }
            P.tile_cu[grp] = (int32_t)tiles;
            valid = valid && tiles == D.score_tiles;
        }
        *P.status = valid ? 0 : (int32_t)FP2_STATUS_BAD_SEQLENS;
        *P.meta_valid = valid;
        s_valid = valid;
    }
    __syncthreads();
    if (s_valid) {
        // the threshold's item counter, the CSR segment counts and the e4m3
        // means' chunk maxima start from zero
        const int64_t n_seg = (D.R + kCsrRows - 1) / kCsrRows, n_sup = (D.R + kCsrSup - 1) / kCsrSup;
        for (int64_t c = threadIdx.x; c < n_seg; c += blockDim.x) P.csr_seg[c] = 0;
        for (int64_t c = threadIdx.x; c < n_sup; c += blockDim.x) P.csr_sup[c] = 0;
        if (threadIdx.x == 0) *P.thr_next = 0;
        for (int64_t c = threadIdx.x; c < 2 * D.NB * D.Hkv; c += blockDim.x) P.mean_amax[c] = 0u;
        meta_maps(D, S, cu_seqlens, page_table, P);
    }
    // k_meta may run beside the pooling kernel launched before it (which
    // needs none of its outputs); it completes only after that kernel, so
    // the kernels after it see both
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Block -> sequence and scoring-group maps, page-id checks, the schedule.
__device__ void meta_maps(const Dims& D, const SchedDims& S, const int32_t* __restrict__ cu_seqlens,
                          const int32_t* __restrict__ page_table, const PlanPtrs& P) {
    for (int s = 0; s < D.n_seqs; ++s) {
        const int b0 = P.cu_blocks[s], b1 = P.cu_blocks[s + 1];
        for (int b = b0 + threadIdx.x; b < b1; b += blockDim.x) P.block_seq[b] = s;
        const int g0 = P.group_cu[s], g1 = P.group_cu[s + 1];
        for (int c = g0 + threadIdx.x; c < g1; c += blockDim.x) P.group_seq[c] = s;
        if (D.page_size) {
            const int np = (cu_seqlens[s + 1] - cu_seqlens[s] + 63) / 64;
            for (int pg = threadIdx.x; pg < np; pg += blockDim.x) {
                const int id = page_table[(int64_t)s * D.pt_stride + pg];
                if (id < 0 || id >= D.num_pages) atomicOr(P.status, (int32_t)FP2_STATUS_BAD_PAGE);
            }
        }
    }
    __syncthreads();
    build_schedule(D, S, P);
}

// ---------------------------------------------------------------------------
// pool: block sums in float64 (one 16-byte column chunk per thread)
// ---------------------------------------------------------------------------

constexpr int kPoolThreads = 128;
constexpr int kPoolUnroll = 8;

__device__ __forceinline__ void accum8(double (&acc)[8], uint4 x) {
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        acc[2 * e] += (double)__uint_as_float(w[e] << 16);
        acc[2 * e + 1] += (double)__uint_as_float(w[e] & 0xFFFF0000u);
    }
}

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// Eight e4m3 codes (8 bytes) added to eight float64 sums; e4m3 -> f16 -> f32
// are exact conversions.
__device__ __forceinline__ void accum8_e4m3(double (&acc)[8], uint2 x) {
    const uint32_t w[2] = {x.x, x.y};
#pragma unroll
    for (int e = 0; e < 2; ++e) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            float lo, hi;
            unpack_e4m3x2(static_cast<uint16_t>(w[e] >> (16 * h)), lo, hi);
            acc[4 * e + 2 * h] += (double)lo;
            acc[4 * e + 2 * h + 1] += (double)hi;
        }
    }
}

__device__ __forceinline__ uint2 ld_stream8(const uint2* p) {
    uint2 r;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];" : "=r"(r.x), "=r"(r.y) : "l"(p));
    return r;
}

__device__ __forceinline__ double warp_sum_d(double x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

__device__ __forceinline__ float round_up_f(double x) {
    // a float not below x (x >= 0)
    float f = (float)x;
    if ((double)f < x) f = nextafterf(f, FLT_MAX);
    return f * (1.0f + 1.0f / 1048576.0f);
}

// The error bound of a tensor-core score.  With q~ = tf32(Qbar_h) and
// k~ = tf32(Kbar) the MMA's operands (exact products, fp32 sums), and the
// score x = fl(fl(q~ . k~) / sqrt d):
//   |Qbar_h . Kbar - q~ . k~| <= |Qbar_h - q~| |Kbar| + |q~| |Kbar - k~|   (Cauchy-Schwarz)
//   |fl(q~ . k~) - q~ . k~|   <= d 2^-23 |q~| |k~|                          (fp32 sums)
//   the division by sqrt d     <= 2^-22 |q~| |k~|                           (two roundings)
// and |q~| <= |Qbar_h| + |Qbar_h - q~|, |k~| <= |Kbar| + |Kbar - k~|, so over
// a row's G heads |x - Qbar . Kbar / sqrt d| <= A kn_j + B kr_j with
//   A = max_h |Qbar_h - q~| / sqrt d,  B = (max_h |Qbar_h| + that) / sqrt d,
//   kn_j = |Kbar_j|,  kr_j = |Kbar_j - k~_j| + c_d (|Kbar_j| + |Kbar_j - k~_j|),
//   c_d = d 2^-23 + 2^-22.
// The residual norms are those of the actual rounding, typically a few times
// below the worst case 2^-11 |.|, which keeps the band of undecided blocks narrow.
__device__ __forceinline__ float kres_bound(double kn, double kr, int d) {
    const double c_d = (double)d * 0x1p-23 + 0x1p-22;
    return round_up_f(kr + c_d * (kn + kr));
}

// Sequence of global block b, its block index i, and its token offsets.
// BYVAL: from the host-computed map passed by value (the pool then needs no
// device-side map and can run before k_meta); otherwise from k_meta's maps.
struct BlockLoc {
    int s, i;
    int64_t tok0;   // first K/V token of the sequence
    int64_t qtok0;  // q token of position 0 of the sequence (chunked: cu_q - q_off)
    int L, q_off;
};

template <bool BYVAL>
__device__ __forceinline__ BlockLoc locate_block(const Dims& D, const SeqMap& M, const PlanPtrs& P,
                                                 const int32_t* __restrict__ cu_seqlens, int64_t b) {
    BlockLoc r;
    if (BYVAL) {
        int lo = 0, hi = M.n - 1;   // the last s with cu_blocks[s] <= b
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (M.cu_blocks[mid] <= b) lo = mid;
            else hi = mid - 1;
        }
        r.s = lo;
        r.i = (int)(b - M.cu_blocks[lo]);
        r.tok0 = M.cu_tok[lo];
        r.L = M.cu_tok[lo + 1] - M.cu_tok[lo];
        r.q_off = M.q_off[lo];
        r.qtok0 = (int64_t)M.cu_q[lo] - r.q_off;
    } else {
        r.s = P.block_seq[b];
        r.i = (int)(b - P.cu_blocks[r.s]);
        r.tok0 = cu_seqlens[r.s];
        r.L = cu_seqlens[r.s + 1] - cu_seqlens[r.s];
        r.q_off = P.cu_q ? P.q_off[r.s] : 0;
        r.qtok0 = P.cu_q ? (int64_t)P.cu_q[r.s] - r.q_off : r.tok0;
    }
    return r;
}

// Block means of Q, K and V.  KV8: K and V are e4m3 codes with one fp32 scale
// per (block, kv-head) (an FP8 KV cache); their means are the means of the
// codes times the scale.  CHUNK: q holds a chunk of each sequence (positions
// q_off .. L - 1), so a query block's mean covers only its chunk positions.
// BYVAL: block -> sequence from the map passed by value (see locate_block);
// the kernel then reads only token rows inside [0, T) (or [0, Tq) of q), so a
// cu_seqlens that disagrees with the host sizes (k_meta flags it) cannot make
// it read out of bounds.  NORMS: also writes |Kbar| per (block, kv-head) and
// the largest |Qbar| over each kv-head's G query heads (both rounded up), the
// threshold's error-bound inputs; needs the G heads of a group inside one CTA.
template <bool KV8, bool CHUNK, bool BYVAL, bool NORMS>
__global__ void __launch_bounds__(kPoolThreads)
k_pool(Dims D, SeqMap M, int64_t Tq, const int32_t* __restrict__ cu_seqlens,
       const int32_t* __restrict__ page_table, const uint16_t* __restrict__ q,
       const void* __restrict__ k, const void* __restrict__ v, const float* __restrict__ k_scale,
       const float* __restrict__ v_scale, const float* __restrict__ prev_kbar,
       const float* __restrict__ prev_vbar, PlanPtrs P, WsPtrs W) {
    // the next kernel (k_meta) may start while the pool runs: it reads none
    // of the pool's outputs and waits for the pool before it completes
    if (BYVAL) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (!BYVAL && !*P.meta_valid) return;
    const int vec = blockIdx.y * kPoolThreads + threadIdx.x;   // 8-element column chunk
    const int d = D.d;
    const int qcols = D.Hq * d, kvcols = D.Hkv * d;
    const int col = vec * 8;
    const bool active = col < qcols + 2 * kvcols;
    const int64_t b = blockIdx.x;
    const BlockLoc loc = locate_block<BYVAL>(D, M, P, cu_seqlens, b);
    const int s = loc.s;
    int64_t tok0 = loc.tok0;
    const int L = loc.L;
    int t_begin = loc.i * D.B;
    int t_end = min(t_begin + D.B, L);

    int which = 0, head = 0, e0 = 0;
    if (col < qcols) { which = 0; head = col / d; e0 = col % d; }
    else if (col < qcols + kvcols) { which = 1; head = (col - qcols) / d; e0 = (col - qcols) % d; }
    else { which = 2; head = (col - qcols - kvcols) / d; e0 = (col - qcols - kvcols) % d; }
    int64_t tok_lim = D.T;   // rows of the tensor read
    if (which == 0) {
        tok_lim = Tq;
        if (CHUNK) {
            // a chunk's queries: positions q_off .. L - 1 are q tokens cu_q[s] ..
            t_begin = max(t_begin, loc.q_off);
            tok0 = loc.qtok0;
        }
    }
    if (BYVAL) {
        // keep every row read inside the tensor, whatever cu_seqlens holds
        if ((int64_t)t_begin < -tok0) t_begin = (int)(-tok0);
        if ((int64_t)t_end > tok_lim - tok0) t_end = (int)(tok_lim - tok0);
    }

    double acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.0;
    // chunked prefill with the caller's means of the blocks wholly before the
    // chunk: those K / V means are copied, not pooled from K and V again
    const float* prev = which == 1 ? prev_kbar : prev_vbar;
    const bool reuse = CHUNK && which != 0 && prev && (loc.i + 1) * D.B <= loc.q_off;

    if (!active) {
        // no column: only takes part in the CTA's barrier below
    } else if (reuse) {
        const float* src = prev + (b * D.Hkv + head) * d + e0;
        const float4 a = __ldg(reinterpret_cast<const float4*>(src));
        const float4 c = __ldg(reinterpret_cast<const float4*>(src + 4));
        const float f[8] = {a.x, a.y, a.z, a.w, c.x, c.y, c.z, c.w};
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = (double)f[e];   // the means themselves
    } else if (KV8 && which != 0) {
        // e4m3 K / V, contiguous [T, Hkv, d] or paged [P, 64, Hkv, d]
        const uint8_t* base = static_cast<const uint8_t*>(which == 1 ? k : v);
        const int64_t stride = (int64_t)D.Hkv_str * d / 8;   // uint2 per token
        if (D.page_size == 0) {
            const uint2* p = reinterpret_cast<const uint2*>(base + ((tok0 + t_begin) * D.Hkv_str + head) * d + e0);
            int t = t_begin;
            for (; t + kPoolUnroll <= t_end; t += kPoolUnroll) {
                uint2 x[kPoolUnroll];
#pragma unroll
                for (int u = 0; u < kPoolUnroll; ++u) x[u] = ld_stream8(p + u * stride);
#pragma unroll
                for (int u = 0; u < kPoolUnroll; ++u) accum8_e4m3(acc, x[u]);
                p += kPoolUnroll * stride;
            }
            for (; t < t_end; ++t) {
                accum8_e4m3(acc, ld_stream8(p));
                p += stride;
            }
        } else {
            for (int t = t_begin; t < t_end; t += 64) {
                const int id = page_table[(int64_t)s * D.pt_stride + t / 64];
                const int n = min(64, t_end - t);
                if (id < 0 || id >= D.num_pages) continue;   // recorded by k_meta; reads as zeros
                const uint2* p = reinterpret_cast<const uint2*>(base + ((int64_t)id * 64 * D.Hkv_str + head) * d + e0);
                for (int u = 0; u < n; ++u) accum8_e4m3(acc, ld_stream8(p + u * stride));
            }
        }
        const double sc = (double)(which == 1 ? k_scale : v_scale)[b * D.Hkv + head];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] *= sc;
    } else if (which == 0 || D.page_size == 0) {
        const uint16_t* base = which == 0 ? q : static_cast<const uint16_t*>(which == 1 ? k : v);
        const int H = which == 0 ? D.Hq_str : D.Hkv_str;   // heads per token of the tensor
        const uint4* p = reinterpret_cast<const uint4*>(base + ((tok0 + t_begin) * H + head) * d + e0);
        const int64_t stride = (int64_t)H * d / 8;   // uint4 per token
        int t = t_begin;
        for (; t + kPoolUnroll <= t_end; t += kPoolUnroll) {
            uint4 x[kPoolUnroll];
#pragma unroll
            for (int u = 0; u < kPoolUnroll; ++u) x[u] = ld_stream(p + u * stride);
#pragma unroll
            for (int u = 0; u < kPoolUnroll; ++u) accum8(acc, x[u]);
            p += kPoolUnroll * stride;
        }
        for (; t < t_end; ++t) {
            accum8(acc, ld_stream(p));
            p += stride;
        }
    } else {
        // paged pool [num_pages, 64, Hkv, d]; blocks start on page boundaries (B % 64 == 0)
        const uint16_t* pool = static_cast<const uint16_t*>(which == 1 ? k : v);
        const int64_t stride = (int64_t)D.Hkv_str * d / 8;
        for (int t = t_begin; t < t_end; t += 64) {
            const int id = page_table[(int64_t)s * D.pt_stride + t / 64];
            const int n = min(64, t_end - t);
            if (id < 0 || id >= D.num_pages) continue;   // recorded by k_meta; reads as zeros
            const uint4* p = reinterpret_cast<const uint4*>(pool + ((int64_t)id * 64 * D.Hkv_str + head) * d + e0);
            int u0 = 0;
            for (; u0 + kPoolUnroll <= n; u0 += kPoolUnroll) {
                uint4 x[kPoolUnroll];
#pragma unroll
                for (int u = 0; u < kPoolUnroll; ++u) x[u] = ld_stream(p + (u0 + u) * stride);
#pragma unroll
                for (int u = 0; u < kPoolUnroll; ++u) accum8(acc, x[u]);
            }
            for (; u0 < n; ++u0) accum8(acc, ld_stream(p + u0 * stride));
        }
    }

    // (a query block below a chunk has no query: its mean is left zero)
    const double inv_n = reuse ? 1.0 : t_end > t_begin ? 1.0 / (double)(t_end - t_begin) : 0.0;
    double m[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) m[e] = acc[e] * inv_n;
    if (active && which == 0) {
        double* dst = W.qbar64 + (b * D.Hq + head) * d + e0;
#pragma unroll
        for (int e = 0; e < 8; e += 2) *reinterpret_cast<double2*>(dst + e) = make_double2(m[e], m[e + 1]);
        // the scorer's operand: the means rounded to tf32
        float* d32 = W.qbar32 + (b * D.Hq + head) * d + e0;
        *reinterpret_cast<float4*>(d32) = make_float4(round_tf32((float)m[0]), round_tf32((float)m[1]),
                                                      round_tf32((float)m[2]), round_tf32((float)m[3]));
        *reinterpret_cast<float4*>(d32 + 4) = make_float4(round_tf32((float)m[4]), round_tf32((float)m[5]),
                                                          round_tf32((float)m[6]), round_tf32((float)m[7]));
    } else if (active) {
        const int64_t off = (b * D.Hkv + head) * d + e0;
        float* f32 = (which == 1 ? P.kbar : P.vbar) + off;
        uint16_t* h16 = (which == 1 ? P.kbar16 : P.vbar16) + off;
        float4 f0 = make_float4((float)m[0], (float)m[1], (float)m[2], (float)m[3]);
        float4 f1 = make_float4((float)m[4], (float)m[5], (float)m[6], (float)m[7]);
        *reinterpret_cast<float4*>(f32) = f0;
        *reinterpret_cast<float4*>(f32 + 4) = f1;
        uint4 hb;
        hb.x = pack_bf16x2(f0.x, f0.y);
        hb.y = pack_bf16x2(f0.z, f0.w);
        hb.z = pack_bf16x2(f1.x, f1.y);
        hb.w = pack_bf16x2(f1.z, f1.w);
        *reinterpret_cast<uint4*>(h16) = hb;
        if (which == 1) {
            double* dst = W.kbar64 + off;
#pragma unroll
            for (int e = 0; e < 8; e += 2) *reinterpret_cast<double2*>(dst + e) = make_double2(m[e], m[e + 1]);
            float* tf = W.kbar_tf + off;
            *reinterpret_cast<float4*>(tf) = make_float4(round_tf32(f0.x), round_tf32(f0.y),
                                                         round_tf32(f0.z), round_tf32(f0.w));
            *reinterpret_cast<float4*>(tf + 4) = make_float4(round_tf32(f1.x), round_tf32(f1.y),
                                                             round_tf32(f1.z), round_tf32(f1.w));
        }
    }
    if (NORMS) {
        // |mean|^2 and |mean - tf32(mean)|^2 of this thread's head: the d / 8
        // threads of a head are consecutive lanes of one warp (d / 8 in {8, 16})
        double sq = 0.0, rq = 0.0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            sq = fma(m[e], m[e], sq);
            const double rr = m[e] - (double)round_tf32((float)m[e]);
            rq = fma(rr, rr, rq);
        }
        const int tph = d / 8;
        for (int o = tph / 2; o > 0; o >>= 1) {
            sq += __shfl_xor_sync(0xffffffffu, sq, o);
            rq += __shfl_xor_sync(0xffffffffu, rq, o);
        }
        const bool lead = active && (vec % tph) == 0;
        if (lead && which == 1) {
            W.kb2[(int64_t)head * D.NB + b] = make_float2(round_up_f(sqrt(sq)), kres_bound(sqrt(sq), sqrt(rq), d));
        }
        // the largest over the G query heads of a kv-head: the group's heads
        // lie in this CTA (G d divides the CTA's 1024 columns)
        __shared__ double head_sq[kPoolThreads], head_rq[kPoolThreads];
        const int hl = threadIdx.x / tph;   // head slot within the CTA
        if (lead) {
            head_sq[hl] = sq;
            head_rq[hl] = rq;
        }
        __syncthreads();
        if (lead && which == 0 && head % D.G == 0) {
            double mx = 0.0, mr = 0.0;
            for (int u = 0; u < D.G; ++u) {
                mx = fmax(mx, head_sq[hl + u]);
                mr = fmax(mr, head_rq[hl + u]);
            }
            W.qnorm[b * D.Hkv + head / D.G] = round_up_f(sqrt(mx));
            W.qres[b * D.Hkv + head / D.G] = round_up_f(sqrt(mr));
        }
    }
}

// ---------------------------------------------------------------------------
// norms: one warp per (block, kv-head)
// ---------------------------------------------------------------------------

__global__ void k_norms(Dims D, PlanPtrs P, WsPtrs W) {
    if (!*P.meta_valid) return;
    const int64_t wid = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (wid >= D.NB * D.Hkv) return;
    const int64_t b = wid / D.Hkv;
    const int g = (int)(wid % D.Hkv);
    const int d = D.d;
    // |mean|^2 and |mean - tf32(mean)|^2 (tf32 of the fp32 mean, the scorer's operand)
    double kk = 0.0, kr = 0.0;
    const double* kp = W.kbar64 + (b * D.Hkv + g) * d;
    for (int e = lane; e < d; e += 32) {
        kk += kp[e] * kp[e];
        const double rr = kp[e] - (double)round_tf32((float)kp[e]);
        kr += rr * rr;
    }
    kk = warp_sum_d(kk);
    kr = warp_sum_d(kr);
    double qmax = 0.0, rmax = 0.0;
    for (int hl = 0; hl < D.G; ++hl) {
        const double* qp = W.qbar64 + (b * D.Hq + (int64_t)g * D.G + hl) * d;
        double qq = 0.0, qr = 0.0;
        for (int e = lane; e < d; e += 32) {
            qq += qp[e] * qp[e];
            const double rr = qp[e] - (double)round_tf32((float)qp[e]);
            qr += rr * rr;
        }
        qq = warp_sum_d(qq);
        qr = warp_sum_d(qr);
        qmax = fmax(qmax, qq);
        rmax = fmax(rmax, qr);
    }
    if (lane == 0) {
        W.kb2[(int64_t)g * D.NB + b] = make_float2(round_up_f(sqrt(kk)), kres_bound(sqrt(kk), sqrt(kr), d));
        W.qnorm[wid] = round_up_f(sqrt(qmax));
        W.qres[wid] = round_up_f(sqrt(rmax));
    }
}

// ---------------------------------------------------------------------------
// score: block scores of every (row, visible key block) on the tensor cores
// ---------------------------------------------------------------------------

// Tensor-core scores.  A tile is (sequence, kv-head, group of 128 / G query
// blocks, chunk of kScoreKeys key blocks) inside the causal triangle; the
// tiles of all row groups are numbered through tile_cu and a persistent CTA
// per SM walks them.  Per tile, the 128 query vectors (the G heads of each
// block of the group) and the 128 key block means, both rounded to tf32, are
// TMA-loaded as 128-byte-swizzled K-major tiles and multiplied by tcgen05 MMAs
// of kind::tf32 (M = N = 128, K = 8 per instruction) into tensor memory; four
// warps read the dot products back, stage them in shared memory, and take the
// maximum over each block's G heads.  With both operands exact tf32 values
// the products are exact and a dot product is within
//   (2 * 2^-11 + d 2^-23) |Qbar| |Kbar|
// of the one of the float64 means (tf32 rounding of both operands, fp32
// accumulation); the threshold kernel uses the tighter bound of kres_bound,
// from the norms of the actual rounding residuals, and re-scores in float64
// every block it cannot decide.
constexpr int kScoreTcThreads = 160;  // warps 0-3: epilogue (TMEM lanes); warp 4: TMA + MMA

template <int HD>
struct ScoreTcCfg {
    static constexpr int kAtoms = HD * 4 / 128;          // 128-byte atoms per fp32 row
    static constexpr int kAtomBytes = 128 * 128;         // one atom column of 128 rows
    static constexpr int kTileBytes = kAtoms * kAtomBytes;
    static constexpr int kDotsBytes = 128 * (kScoreKeys + 1) * 4;
    static constexpr int kSmem = (2 * kTileBytes > kDotsBytes ? 2 * kTileBytes : kDotsBytes) + 1024;
};

template <int HD>
__global__ void __launch_bounds__(kScoreTcThreads)
k_score_tc(Dims D, PlanPtrs P, WsPtrs W, const __grid_constant__ CUtensorMap tm_q,
           const __grid_constant__ CUtensorMap tm_k) {
    using C = ScoreTcCfg<HD>;
    // a programmatic dependent of the kernel before it: everything before is
    // complete once the wait returns; the threshold after it may be launched
    // early (it waits for this kernel before reading anything)
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (!*P.meta_valid) return;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    __shared__ uint64_t bar_full, bar_done;
    __shared__ uint32_t tmem_base;
    __shared__ volatile int abort_flag;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int RI = D.rows_per_group;
    const int G = D.G;
    const int n_groups = P.group_cu[D.n_seqs];

    if (tid == 0) {
        mbar_init(&bar_full, 1);
        mbar_init(&bar_done, 1);
        abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        fence_proxy_async_smem();
    }
    if (warp == 0) tmem_alloc(&tmem_base, kScoreKeys);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base;
    unsigned char* sa = smem;
    unsigned char* sb = smem + C::kTileBytes;
    float* dots = reinterpret_cast<float*>(smem);   // [128][kScoreKeys + 1], after the MMAs
    const float inv_sqrt_d = 1.0f / sqrtf((float)HD);
    const int64_t n_items = D.score_tiles * D.Hkv;
    uint32_t phase = 0;

    for (int64_t w = blockIdx.x; w < n_items; w += gridDim.x, phase ^= 1u) {
        const int g = (int)(w % D.Hkv);
        const int tile = (int)(w / D.Hkv);
        // row group of the tile: the last gi with tile_cu[gi] <= tile
        int lo = 0, hi = n_groups - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (P.tile_cu[mid] <= tile) lo = mid;
            else hi = mid - 1;
        }
        const int gi = lo;
        const int jc = tile - P.tile_cu[gi];
        const int s = P.group_seq[gi];
        const int b0 = P.cu_blocks[s];
        const int nb = P.cu_blocks[s + 1] - b0;
        const int i0 = (gi - P.group_cu[s]) * RI;
        const int i1 = min(i0 + RI, nb);
        const int j0 = jc * kScoreKeys;
        const int j1 = min(j0 + kScoreKeys, i1);
        const int nrows = i1 - i0;

        if (warp == 4 && lane == 0) {
            mbar_arrive_expect_tx(&bar_full, C::kAtoms * (G * RI * 128 + kScoreKeys * 128));
#pragma unroll
            for (int a = 0; a < C::kAtoms; ++a) {
                tma_load_3d(sa + a * C::kAtomBytes, &tm_q, &bar_full, 32 * a, g * G, b0 + i0);
                tma_load_3d(sb + a * C::kAtomBytes, &tm_k, &bar_full, 32 * a, g, b0 + j0);
            }
            if (mbar_wait(&bar_full, phase, &abort_flag, P.status)) {
                tc_fence_after();
                const uint64_t da = smem_desc_sw128(smem_u32(sa), 16, 1024);
                const uint64_t db = smem_desc_sw128(smem_u32(sb), 16, 1024);
                constexpr uint32_t idesc = idesc_tf32(128, kScoreKeys);
#pragma unroll
                for (int kk = 0; kk < HD / 8; ++kk) {
                    const uint32_t off = (kk / 4) * C::kAtomBytes + (kk % 4) * 32;
                    umma_tf32(tmem, da + (off >> 4), db + (off >> 4), idesc, kk > 0 ? 1u : 0u);
                }
                umma_commit(&bar_done);
            } else {
                // the copies may still land: wait for them before leaving
                mbar_wait_drain(&bar_full, phase, P.status);
            }
        }
        if (warp < 4) {
            const bool ok = __all_sync(0xffffffffu, mbar_wait(&bar_done, phase, &abort_flag, P.status));
            if (ok) {
                tc_fence_after();
                const int row = 32 * warp + lane;
#pragma unroll 1
                for (int c = 0; c < kScoreKeys / 32; ++c) {
                    uint32_t r[32];
                    tmem_ld32(tmem + (static_cast<uint32_t>(32 * warp) << 16) + 32 * c, r);
                    tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        dots[row * (kScoreKeys + 1) + 32 * c + e] = __uint_as_float(r[e]);
                }
            } else {
                abort_flag = 1;
            }
        }
        tc_fence_before();
        __syncthreads();
        if (abort_flag) break;
        float* scores = W.scores + (int64_t)g * D.tri_total + P.tri_off[s];
        for (int idx = tid; idx < nrows * kScoreKeys; idx += kScoreTcThreads) {
            const int ri = idx / kScoreKeys, jj = idx % kScoreKeys;
            const int i = i0 + ri, j = j0 + jj;
            if (j <= i && j < j1) {
                const float* col = dots + (ri * G) * (kScoreKeys + 1) + jj;
                float best = col[0];
                for (int hl = 1; hl < G; ++hl) best = fmaxf(best, col[hl * (kScoreKeys + 1)]);
                if (FP2_CHECK(P.tri_off[s] + (int64_t)i * (i + 1) / 2 + j < D.tri_total, P.status))
                    scores[(int64_t)i * (i + 1) / 2 + j] = best * inv_sqrt_d;
            }
        }
        __syncthreads();   // the staged dots are read before the next tile's copies land
        tc_fence_after();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kScoreKeys);
    }
}

// Pipelined tensor-core scores (G a power of two, at most 32).  A persistent CTA per SM takes
// work items (row group of 128 / G query blocks, kv-head), the row groups of
// a sequence from the last (longest rows) down, kv-heads inner, one item per
// CTA per pass over the grid (odd passes from the other end).  Roles:
//   warp 4  TMA: the item's 128 query vectors (tf32 values in fp32) once,
//           then its 128-key-block chunks into a 2-slot ring;
//   warp 5  MMA: per chunk 16 (d = 128) tcgen05 kind::tf32 MMAs
//           (M = N = 128, K = 8) into one of two 128-column TMEM accumulators;
//   warps 0-3  epilogue: each thread reads its query vector's 128 dot
//           products from TMEM, the G heads of a block (G adjacent lanes)
//           take their maximum by shuffles, and the block's first lane
//           stores the scores j <= i of that chunk.
// The loads of chunk c + 1 and its MMAs overlap the epilogue of chunk c.
// Products and error bound as for k_score_tc.
constexpr int kScorePThreads = 192;

template <int HD>
struct ScorePCfg {
    static constexpr int kAtoms = HD * 4 / 128;          // 128-byte atoms per fp32 row
    static constexpr int kAtomBytes = 128 * 128;         // one atom column of 128 rows
    static constexpr int kTileBytes = kAtoms * kAtomBytes;
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = kTileBytes;             // two K slots
    static constexpr int kSmem = 3 * kTileBytes + 1024;
};

struct ScoreItem {
    int g, s, b0, nb, i0, i1, n_chunks;
};

__device__ __forceinline__ ScoreItem score_item(const Dims& D, const PlanPtrs& P, int64_t w,
                                                int n_groups) {
    const int64_t n_items = (int64_t)n_groups * D.Hkv;
    const int64_t pass = w / gridDim.x;
    const int64_t o = (pass & 1) ? pass * gridDim.x + (gridDim.x - 1 - blockIdx.x) : w;
    ScoreItem it;
    it.n_chunks = 0;
    if (o >= n_items) return it;
    const int gi = n_groups - 1 - (int)(o / D.Hkv);
    it.g = (int)(o % D.Hkv);
    it.s = P.group_seq[gi];
    it.b0 = P.cu_blocks[it.s];
    it.nb = P.cu_blocks[it.s + 1] - it.b0;
    it.i0 = (gi - P.group_cu[it.s]) * D.rows_per_group;
    it.i1 = min(it.i0 + D.rows_per_group, it.nb);
    it.n_chunks = (it.i1 - 1) / kScoreKeys + 1;
    return it;
}

template <int HD, int GQ>
__global__ void __launch_bounds__(kScorePThreads, 1)
k_score_pipe(Dims D, PlanPtrs P, WsPtrs W, const __grid_constant__ CUtensorMap tm_q,
             const __grid_constant__ CUtensorMap tm_k) {
    using C = ScorePCfg<HD>;
    // a programmatic dependent of the kernel before it: everything before is
    // complete once the wait returns; the threshold after it may be launched
    // early (it waits for this kernel before reading anything)
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (!*P.meta_valid) return;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    __shared__ uint64_t q_full, q_empty, k_full[2], k_empty[2], acc_full[2], acc_empty[2], drain;
    __shared__ uint32_t tmem_base;
    __shared__ volatile int abort_flag;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n_groups = P.group_cu[D.n_seqs];
    const int64_t n_items = (int64_t)n_groups * D.Hkv;
    const int64_t n_slots = (n_items + gridDim.x - 1) / gridDim.x * gridDim.x;

    if (tid == 0) {
        mbar_init(&q_full, 1);
        mbar_init(&q_empty, 1);
        mbar_init(&drain, 1);
        for (int u = 0; u < 2; ++u) {
            mbar_init(&k_full[u], 1);
            mbar_init(&k_empty[u], 1);
            mbar_init(&acc_full[u], 1);
            mbar_init(&acc_empty[u], 4);
        }
        abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        fence_proxy_async_smem();
    }
    if (warp == 5) tmem_alloc(&tmem_base, 2 * kScoreKeys);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base;

    if (warp == 4) {
        if (lane == 0) {
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_k);
            uint32_t qn = 0, kn = 0;   // Q loads, K chunk loads issued
            uint32_t kuse[2] = {0, 0};  // loads issued into each K slot
            for (int64_t w = blockIdx.x; w < n_slots; w += gridDim.x) {
                const ScoreItem it = score_item(D, P, w, n_groups);
                if (it.n_chunks == 0) continue;
                if (!mbar_wait(&q_empty, (qn & 1) ^ 1, &abort_flag, P.status)) break;
                ++qn;
                mbar_arrive_expect_tx(&q_full, C::kAtoms * kScoreQV * 128);
#pragma unroll
                for (int a = 0; a < C::kAtoms; ++a)
                    tma_load_3d(smem + C::kOffQ + a * C::kAtomBytes, &tm_q, &q_full, 32 * a, it.g * D.G,
                                it.b0 + it.i0);
                bool ok = true;
                for (int c = 0; c < it.n_chunks && ok; ++c, ++kn) {
                    const int slot = kn & 1;
                    if (!mbar_wait(&k_empty[slot], ((kn >> 1) & 1) ^ 1, &abort_flag, P.status)) {
                        ok = false;
                        break;
                    }
                    ++kuse[slot];
                    mbar_arrive_expect_tx(&k_full[slot], C::kAtoms * kScoreKeys * 128);
#pragma unroll
                    for (int a = 0; a < C::kAtoms; ++a)
                        tma_load_3d(smem + C::kOffK + slot * C::kTileBytes + a * C::kAtomBytes, &tm_k,
                                    &k_full[slot], 32 * a, it.g, it.b0 + kScoreKeys * c);
                }
                if (!ok) break;
            }
            // let the copies in flight land before the CTA may exit
            if (qn) mbar_wait_drain(&q_full, (qn - 1) & 1, P.status);
            for (int u = 0; u < 2; ++u)
                if (kuse[u]) mbar_wait_drain(&k_full[u], (kuse[u] - 1) & 1, P.status);
        }
    } else if (warp == 5) {
        if (lane == 0) {
            const uint64_t dq = smem_desc_sw128(smem_u32(smem + C::kOffQ), 16, 1024);
            constexpr uint32_t idesc = idesc_tf32(128, kScoreKeys);
            uint32_t qn = 0, kn = 0, an = 0;
            for (int64_t w = blockIdx.x; w < n_slots; w += gridDim.x) {
                const ScoreItem it = score_item(D, P, w, n_groups);
                if (it.n_chunks == 0) continue;
                if (!mbar_wait(&q_full, qn & 1, &abort_flag, P.status)) break;
                ++qn;
                bool ok = true;
                for (int c = 0; c < it.n_chunks; ++c, ++kn, ++an) {
                    const int slot = kn & 1, buf = an & 1;
                    if (!mbar_wait(&k_full[slot], (kn >> 1) & 1, &abort_flag, P.status) ||
                        !mbar_wait(&acc_empty[buf], ((an >> 1) & 1) ^ 1, &abort_flag, P.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t dk = smem_desc_sw128(smem_u32(smem + C::kOffK + slot * C::kTileBytes), 16, 1024);
#pragma unroll
                    for (int kk = 0; kk < HD / 8; ++kk) {
                        const uint32_t off = (kk / 4) * C::kAtomBytes + (kk % 4) * 32;
                        umma_tf32(tmem + buf * kScoreKeys, dq + (off >> 4), dk + (off >> 4), idesc,
                                  kk > 0 ? 1u : 0u);
                    }
                    umma_commit(&k_empty[slot]);
                    umma_commit(&acc_full[buf]);
                }
                if (!ok) break;
                umma_commit(&q_empty);
            }
            // every MMA issued above completes before the CTA may exit
            umma_commit(&drain);
            mbar_wait_drain(&drain, 0, P.status);
        }
    } else {
        // epilogue warps 0-3: thread = query vector (block ri, head hl) of the item;
        // the block's first lane also keeps the row's largest lower and upper
        // bound of any score, sc_j -/+ C |Qbar|max |Kbar_j| (the threshold's
        // first pass, done here while the scores are in registers)
        const float inv_sqrt_d = 1.0f / sqrtf((float)HD);
        const double inv_sqrt_d64 = 1.0 / sqrt((double)HD);
        constexpr int G = GQ;   // query heads per kv-head (a power of two, at most 32)
        const int row = 32 * warp + lane;
        const int ri = row / G, hl = row % G;
        uint32_t an = 0;
        for (int64_t w = blockIdx.x; w < n_slots; w += gridDim.x) {
            const ScoreItem it = score_item(D, P, w, n_groups);
            if (it.n_chunks == 0) continue;
            const int i = it.i0 + ri;
            // the G lanes of a block share its columns: lane hl takes columns hl, hl + G, ...
            const bool row_ok = i < it.i1;
            float* sc_row = W.scores + (int64_t)it.g * D.tri_total + P.tri_off[it.s] + (int64_t)i * (i + 1) / 2;
            const float2* kb2 = W.kb2 + (int64_t)it.g * D.NB + it.b0;
            // the row's bound coefficients A, B (see kres_bound), rounded up (the
            // bounds below only need to enclose the float64 ones: they are
            // widened before they are stored)
            float A = 0.f, B = 0.f;
            if (row_ok) {
                const int64_t qi = (int64_t)(it.b0 + i) * D.Hkv + it.g;
                const double qr = W.qres[qi];
                A = round_up_f(qr * inv_sqrt_d64);
                B = round_up_f(((double)W.qnorm[qi] + qr) * inv_sqrt_d64);
            }
            float m_lo = -FLT_MAX, m_hi = -FLT_MAX, e_max = 0.f;
            bool ok = true;
            for (int c = 0; c < it.n_chunks; ++c, ++an) {
                const int buf = an & 1;
                // the chunk's key norms, lane l holding column 32 cc + l of each
                // 32-column part (loaded before the wait, handed out by shuffles)
                constexpr int NCC = kScoreKeys / 32;
                float knr[NCC], krr[NCC];
#pragma unroll
                for (int cc = 0; cc < NCC; ++cc) {
                    const int col = kScoreKeys * c + 32 * cc + lane;
                    const float2 t2 = col < it.nb ? __ldg(kb2 + col) : make_float2(0.f, 0.f);
                    knr[cc] = t2.x;
                    krr[cc] = t2.y;
                }
                if (!__all_sync(0xffffffffu, mbar_wait(&acc_full[buf], (an >> 1) & 1, &abort_flag, P.status))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                // all of the chunk's dot products at once; the accumulator is
                // free for the MMAs two chunks on as soon as they are in registers
                uint32_t r[NCC][32];
#pragma unroll
                for (int cc = 0; cc < NCC; ++cc)
                    tmem_ld32(tmem + (static_cast<uint32_t>(32 * warp) << 16) + buf * kScoreKeys + 32 * cc, r[cc]);
                tmem_ld_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&acc_empty[buf]);
#pragma unroll
                for (int cc = 0; cc < NCC; ++cc) {
                    const int jb = kScoreKeys * c + 32 * cc;
                    // max over the G heads (adjacent lanes) by halving exchanges: at
                    // the step of bit b, lane hl keeps the columns whose bit b is
                    // that of hl, sends its partner (lane ^ b) the others, and keeps
                    // the max of each kept pair in the slot of the column with bit b
                    // clear.  After the steps, slot e0 (a multiple of G) holds the
                    // max for column e0 + hl: 32 - 32 / G shuffles, not 32 log2 G.
#pragma unroll
                    for (int b = G / 2; b >= 1; b >>= 1) {
                        const bool up = (hl & b) != 0;
#pragma unroll
                        for (int c0 = 0; c0 < 32; ++c0) {
                            // slots still in use have every bit of G above b clear
                            if ((c0 & (G - 1) & ~(b - 1)) != 0) continue;
                            const uint32_t lo = r[cc][c0], hi = r[cc][c0 | b];
                            const uint32_t keep = up ? hi : lo, send = up ? lo : hi;
                            const float got = __shfl_xor_sync(0xffffffffu, __uint_as_float(send), b);
                            r[cc][c0] = __float_as_uint(fmaxf(__uint_as_float(keep), got));
                        }
                    }
                    float lo4[4] = {-FLT_MAX, -FLT_MAX, -FLT_MAX, -FLT_MAX};
                    float hi4[4] = {-FLT_MAX, -FLT_MAX, -FLT_MAX, -FLT_MAX};
#pragma unroll
                    for (int e0 = 0; e0 < 32; e0 += G) {
                        // this lane's column of the G columns e0 .. e0 + G - 1
                        const uint32_t v = r[cc][e0];
                        const float knv = __shfl_sync(0xffffffffu, knr[cc], e0 + hl);
                        const float krv = __shfl_sync(0xffffffffu, krr[cc], e0 + hl);
                        const int col = jb + e0 + hl;
                        if (row_ok && col <= i &&
                            FP2_CHECK(sc_row + col < W.scores + D.Hkv * D.tri_total, P.status)) {
                            const float x = __uint_as_float(v) * inv_sqrt_d;
                            sc_row[col] = x;
                            const float err = fmaf(A, knv, B * krv);
                            e_max = fmaxf(e_max, err);
                            lo4[(e0 / G) & 3] = fmaxf(lo4[(e0 / G) & 3], x - err);
                            hi4[(e0 / G) & 3] = fmaxf(hi4[(e0 / G) & 3], x + err);
                        }
                    }
                    m_lo = fmaxf(m_lo, fmaxf(fmaxf(lo4[0], lo4[1]), fmaxf(lo4[2], lo4[3])));
                    m_hi = fmaxf(m_hi, fmaxf(fmaxf(hi4[0], hi4[1]), fmaxf(hi4[2], hi4[3])));
                }
            }
            if (!ok) {
                abort_flag = 1;
                break;
            }
            // the row's bounds over its G lanes' columns
#pragma unroll
            for (int o = 1; o < G; o <<= 1) {
                m_lo = fmaxf(m_lo, __shfl_xor_sync(0xffffffffu, m_lo, o));
                m_hi = fmaxf(m_hi, __shfl_xor_sync(0xffffffffu, m_hi, o));
                e_max = fmaxf(e_max, __shfl_xor_sync(0xffffffffu, e_max, o));
            }
            if (row_ok && hl == 0) {
                // widened by far more than the fp32 rounding of the terms above, so
                // that [m_lo, m_hi] holds the row's float64 maximum
                const double slack = ((double)fabsf(m_lo) + (double)fabsf(m_hi) + (double)e_max) * 0x1p-18 + 1e-30;
                const int64_t r = (int64_t)it.g * D.NB + it.b0 + i;
                W.bounds[2 * r] = (double)m_lo - slack;
                W.bounds[2 * r + 1] = (double)m_hi + slack;
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        tc_fence_after();
        tmem_dealloc(tmem, 2 * kScoreKeys);
    }
}

// float64 score of a key block for a row: max over the group's G heads of
// Qbar_h . Kbar / sqrt(d), from the float64 means (warp-collective).
// qp0: Qbar64 of the row's first head (the G heads follow, HD apart); kp: Kbar64.
// (Not inlined: it is called from several unrolled loops, and a re-score is
// rare -- about two per row -- so one out-of-line copy keeps the threshold
// kernel small.)
template <int HD>
__device__ __noinline__ double score64(const double* __restrict__ qp0, const double* __restrict__ kp,
                                       int G) {
    constexpr int E = HD / 32;   // elements per lane
    const int lane = threadIdx.x & 31;
    double kv[E];
#pragma unroll
    for (int e = 0; e < E; ++e) kv[e] = __ldg(kp + lane + 32 * e);
    double best = -DBL_MAX;
    // four heads at a time: their loads and reductions overlap
    for (int h0 = 0; h0 < G; h0 += 4) {
        double acc[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            acc[u] = 0.0;
            if (h0 + u < G) {
                const double* qp = qp0 + (int64_t)(h0 + u) * HD;
#pragma unroll
                for (int e = 0; e < E; ++e) acc[u] = fma(__ldg(qp + lane + 32 * e), kv[e], acc[u]);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
#pragma unroll
            for (int u = 0; u < 4; ++u) acc[u] += __shfl_xor_sync(0xffffffffu, acc[u], o);
#pragma unroll
        for (int u = 0; u < 4; ++u)
            if (h0 + u < G) best = fmax(best, acc[u]);
    }
    return best / sqrt((double)HD);
}

// ---------------------------------------------------------------------------
// e4m3 codes of the K / V block means for the FP8 correction
// ---------------------------------------------------------------------------
//
// A chunk is the B consecutive blocks of a sequence that one pseudo-key tile
// covers, so a pseudo tile needs a single scale per kv-head:
// scale = absmax / 448 over the chunk's fp32 means (1 when all zero),
// code = e4m3_rne_sat(mean / scale), both in fp32.  The key means get a second
// e4m3 term, lo = e4m3_rne_sat(mean / scale - code), so that the pseudo-key
// logits (one MMA over both terms) carry about 2^-8 relative error instead of
// the 2^-4 of one e4m3 rounding.  Two steps ride on kernels that run anyway:
// the threshold kernel's warps take the chunks' absolute maxima (one item per
// block, atomicMax of the bits of a non-negative float into the chunk's slot),
// the CSR kernel's warps then write the codes and scales (one item per block).

__device__ __forceinline__ uint16_t e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// First block of the chunk that holds block b.
__device__ __forceinline__ int64_t chunk_first(const Dims& D, const PlanPtrs& P, int64_t b) {
    const int b0 = P.cu_blocks[P.block_seq[b]];
    return b0 + (b - b0) / D.B * D.B;
}

// Warp-collective: the K and V means of block b, all kv-heads (Hkv d floats
// each, lane l taking 4 consecutive floats of every 128), visited one float4
// at a time with f(h, k4, v4, lead); the d / 4 lanes of a head form one
// aligned group of lanes (d / 4 in {16, 32}), `lead` is its first lane.
template <typename F>
__device__ __forceinline__ void for_means(const Dims& D, const PlanPtrs& P, int64_t b, int lane, F f) {
    const int d = D.d;
    const int n4 = D.Hkv * d / 4;
    const int lph = d / 4;
    for (int f0 = 0; f0 < n4; f0 += 32) {
        const int f4 = f0 + lane;
        const bool in = f4 < n4;
        const int64_t off = b * D.Hkv * d + 4 * (int64_t)f4;
        const float4 k4 = in ? *reinterpret_cast<const float4*>(P.kbar + off) : make_float4(0.f, 0.f, 0.f, 0.f);
        const float4 v4 = in ? *reinterpret_cast<const float4*>(P.vbar + off) : make_float4(0.f, 0.f, 0.f, 0.f);
        f(in ? 4 * f4 / d : -1, off, k4, v4, (lane % lph) == 0, lph);
    }
}

__device__ __forceinline__ float absmax4(float4 x) {
    return fmaxf(fmaxf(fabsf(x.x), fabsf(x.y)), fmaxf(fabsf(x.z), fabsf(x.w)));
}

// Step 1 (a threshold-kernel item): block b's absolute maxima into its chunk's slots.
__device__ __forceinline__ void means_absmax(const Dims& D, const PlanPtrs& P, int64_t b, int lane) {
    const int64_t c0 = chunk_first(D, P, b);
    for_means(D, P, b, lane, [&](int h, int64_t, float4 k4, float4 v4, bool lead, int lph) {
        float mk = absmax4(k4), mv = absmax4(v4);
        for (int o = lph / 2; o > 0; o >>= 1) {
            mk = fmaxf(mk, __shfl_xor_sync(0xffffffffu, mk, o));
            mv = fmaxf(mv, __shfl_xor_sync(0xffffffffu, mv, o));
        }
        if (lead && h >= 0) {
            atomicMax(P.mean_amax + (c0 * D.Hkv + h) * 2, __float_as_uint(mk));
            atomicMax(P.mean_amax + (c0 * D.Hkv + h) * 2 + 1, __float_as_uint(mv));
        }
    });
}

// Step 2 (a CSR-kernel item): block b's codes from its chunk's maxima; the
// chunk's first block also writes the chunk's scales.
__device__ __forceinline__ void means_codes(const Dims& D, const PlanPtrs& P, int64_t b, int lane) {
    const int64_t c0 = chunk_first(D, P, b);
    for_means(D, P, b, lane, [&](int h, int64_t off, float4 k4, float4 v4, bool lead, int) {
        if (h < 0) return;
        const float mk = __uint_as_float(P.mean_amax[(c0 * D.Hkv + h) * 2]);
        const float mv = __uint_as_float(P.mean_amax[(c0 * D.Hkv + h) * 2 + 1]);
        const float sk = mk > 0.f ? __fdiv_rn(mk, 448.0f) : 1.0f;
        const float sv = mv > 0.f ? __fdiv_rn(mv, 448.0f) : 1.0f;
        if (lead && b == c0) {
            P.kbar_scale[b * D.Hkv + h] = sk;
            P.vbar_scale[b * D.Hkv + h] = sv;
        }
        const float kq[4] = {__fdiv_rn(k4.x, sk), __fdiv_rn(k4.y, sk), __fdiv_rn(k4.z, sk),
                             __fdiv_rn(k4.w, sk)};
        const uint16_t h01 = e4m3x2(kq[0], kq[1]), h23 = e4m3x2(kq[2], kq[3]);
        *reinterpret_cast<uint32_t*>(P.kbar8 + off) = (uint32_t)h01 | ((uint32_t)h23 << 16);
        // second term: the residual of the quotient (exact in fp32, since the
        // e4m3 value is within a factor 2 of it), rounded to e4m3 on its own
        float hv[4];
        unpack_e4m3x2(h01, hv[0], hv[1]);
        unpack_e4m3x2(h23, hv[2], hv[3]);
        *reinterpret_cast<uint32_t*>(P.kbar8lo + off) =
            (uint32_t)e4m3x2(kq[0] - hv[0], kq[1] - hv[1]) |
            ((uint32_t)e4m3x2(kq[2] - hv[2], kq[3] - hv[3]) << 16);
        *reinterpret_cast<uint32_t*>(P.vbar8 + off) =
            (uint32_t)e4m3x2(__fdiv_rn(v4.x, sv), __fdiv_rn(v4.y, sv)) |
            ((uint32_t)e4m3x2(__fdiv_rn(v4.z, sv), __fdiv_rn(v4.w, sv)) << 16);
    });
}

// ---------------------------------------------------------------------------
// threshold: one warp per row, decisions equal to the float64 ones
// ---------------------------------------------------------------------------
//
// The score of block j of a row differs from the exact one by at most
//   e_j = A kn_j + B kr_j
// (kres_bound: A, B per row from its query means, kn_j, kr_j per key block).
// Every block whose score could be the row maximum and every block whose
// score lies within e_j of tau * m is re-scored in float64.
// The loads of a row are issued kThrBatch words (32 blocks each) at a time,
// so a pass over a row of n blocks waits on about n / (32 kThrBatch) round
// trips to L2 rather than n / 32.
constexpr int kThrBatch = 4;

// The error-bound terms of one row.
struct RowBound {
    const float2* kb;  // (|Kbar_j|, kr_j), j = 0 .. i
    double A, B;
    __device__ __forceinline__ double e(float knj, float krj) const { return A * knj + B * krj; }
};

// The decision of one row (warp-collective), given the largest lower bound
// m_lo of its scores: the row maximum in float64 over every block whose upper
// bound reaches m_lo, then keep / drop per block, re-scoring in float64 every
// block within its bound e_j of the threshold.  Writes the mask words
// 0 .. i / 32 and zeroes the rest; adds the kept count to `count`.
template <int HD>
__device__ __forceinline__ void thr_decide(const Dims& D, const WsPtrs& W, const float* sc,
                                           const RowBound& rb, double m_lo, int i, int64_t bi, int b0,
                                           int g, int lane, uint32_t* mask, int& count) {
    const double* q64 = W.qbar64 + (bi * D.Hq + (int64_t)g * D.G) * HD;   // the row's first head
    double m = -DBL_MAX;
#pragma unroll 1
    for (int jb = 0; jb <= i; jb += 32 * kThrBatch) {
        float xs[kThrBatch], ks[kThrBatch], rs[kThrBatch];
#pragma unroll
        for (int u = 0; u < kThrBatch; ++u) {
            const int j = jb + 32 * u + lane;
            xs[u] = j <= i ? __ldg(sc + j) : 0.f;
            const float2 t2 = j <= i ? __ldg(rb.kb + j) : make_float2(0.f, 0.f);
            ks[u] = t2.x;
            rs[u] = t2.y;
        }
#pragma unroll
        for (int u = 0; u < kThrBatch; ++u) {
            const int j = jb + 32 * u + lane;
            uint32_t cb = __ballot_sync(0xffffffffu, j <= i && (double)xs[u] + rb.e(ks[u], rs[u]) >= m_lo);
            while (cb) {
                const int l = __ffs(cb) - 1;
                cb &= cb - 1;
                m = fmax(m, score64<HD>(q64, W.kbar64 + ((int64_t)(b0 + jb + 32 * u + l) * D.Hkv + g) * HD, D.G));
            }
        }
    }
    const double t = D.tau * m;
#pragma unroll 1
    for (int jb = 0; jb <= i; jb += 32 * kThrBatch) {
        float xs[kThrBatch], ks[kThrBatch], rs[kThrBatch];
#pragma unroll
        for (int u = 0; u < kThrBatch; ++u) {
            const int j = jb + 32 * u + lane;
            xs[u] = j <= i ? __ldg(sc + j) : 0.f;
            const float2 t2 = j <= i ? __ldg(rb.kb + j) : make_float2(0.f, 0.f);
            ks[u] = t2.x;
            rs[u] = t2.y;
        }
#pragma unroll
        for (int u = 0; u < kThrBatch; ++u) {
            if (jb + 32 * u > i) break;
            const int j = jb + 32 * u + lane;
            bool keep = false, unsure = false;
            if (j <= i) {
                if (j == 0 || j == i) {
                    keep = true;
                } else {
                    const double e = rb.e(ks[u], rs[u]);
                    const double x = (double)xs[u];
                    if (x - e >= t) keep = true;
                    else if (!(x + e < t)) unsure = true;
                }
            }
            uint32_t ub = __ballot_sync(0xffffffffu, unsure);
            while (ub) {
                const int l = __ffs(ub) - 1;
                ub &= ub - 1;
                const double x64 = score64<HD>(q64, W.kbar64 + ((int64_t)(b0 + jb + 32 * u + l) * D.Hkv + g) * HD, D.G);
                if (lane == l) keep = x64 >= t;
            }
            const uint32_t bits = __ballot_sync(0xffffffffu, keep);
            if (lane == 0) mask[(jb >> 5) + u] = bits;
            count += __popc(bits);
        }
    }
    for (int w = i / 32 + 1 + lane; w < D.mask_words; w += 32) mask[w] = 0u;
}

// One pass over a row of at most 1024 blocks whose score bounds the scorer
// left in W.bounds: the exact maximum m lies in [m_lo, m_hi], so a block is
// kept outright when sc - e >= tau m_hi, dropped outright when
// sc + e < tau m_lo, and otherwise decided once m is known.  The tests run
// in fp32 with every rounding directed against the outright decisions (e,
// sc +/- e and the thresholds they meet rounded up or down as the test
// needs), so a block decided outright is decided as the exact values decide
// it.  The candidates for the maximum (sc + e >= m_lo) are marked on the way
// and re-scored in float64 only when the row has an undecided block.  The
// next 32 kThrBatch scores are loaded while a batch is classified.  Lane l
// keeps the bits of mask word l.
template <int HD>
__device__ __forceinline__ void thr_one_pass(const Dims& D, const WsPtrs& W, const float* sc,
                                             const RowBound& rb, double m_lo, double m_hi, int i,
                                             int64_t bi, int b0, int g, int lane, uint32_t* mask,
                                             int& count) {
    const double* q64 = W.qbar64 + (bi * D.Hq + (int64_t)g * D.G) * HD;   // the row's first head
    const float a_f = __double2float_ru(rb.A), b_f = __double2float_ru(rb.B);
    const float m_lo_f = __double2float_rd(m_lo);
    const float t_lo_f = __double2float_rd(D.tau * m_lo);
    const float t_hi_f = __double2float_ru(D.tau * m_hi);
    uint32_t my_pending = 0, my_keep = 0, my_cand = 0;   // of mask word `lane`
    float xn[kThrBatch], kq[kThrBatch], rq[kThrBatch];
#pragma unroll
    for (int u = 0; u < kThrBatch; ++u) {
        const int j = 32 * u + lane;
        xn[u] = j <= i ? __ldg(sc + j) : 0.f;
        const float2 t2 = j <= i ? __ldg(rb.kb + j) : make_float2(0.f, 0.f);
        kq[u] = t2.x;
        rq[u] = t2.y;
    }
#pragma unroll 1
    for (int jb = 0; jb <= i; jb += 32 * kThrBatch) {
        float xs[kThrBatch], es[kThrBatch];
#pragma unroll
        for (int u = 0; u < kThrBatch; ++u) {
            xs[u] = xn[u];
            es[u] = __fmaf_ru(a_f, kq[u], __fmul_ru(b_f, rq[u]));   // >= e_j
        }
        if (jb + 32 * kThrBatch <= i) {
#pragma unroll
            for (int u = 0; u < kThrBatch; ++u) {
                const int j = jb + 32 * kThrBatch + 32 * u + lane;
                xn[u] = j <= i ? __ldg(sc + j) : 0.f;
                const float2 t2 = j <= i ? __ldg(rb.kb + j) : make_float2(0.f, 0.f);
                kq[u] = t2.x;
                rq[u] = t2.y;
            }
        }
#pragma unroll
        for (int u = 0; u < kThrBatch; ++u) {
            if (jb + 32 * u > i) break;
            const int j = jb + 32 * u + lane;
            const int w = (jb >> 5) + u;
            bool keep = false, pend = false, cand = false;
            if (j <= i) {
                const float hi = __fadd_ru(xs[u], es[u]);   // >= sc + e
                const float lo = __fsub_rd(xs[u], es[u]);   // <= sc - e
                cand = hi >= m_lo_f;
                if (j == 0 || j == i || lo >= t_hi_f) keep = true;
                else if (!(hi < t_lo_f)) pend = true;
            }
            const uint32_t kb = __ballot_sync(0xffffffffu, keep);
            const uint32_t pb = __ballot_sync(0xffffffffu, pend);
            const uint32_t cb = __ballot_sync(0xffffffffu, cand);
            if (lane == w) {
                my_keep = kb;
                my_pending = pb;
                my_cand = cb;
            }
        }
    }
    if (__any_sync(0xffffffffu, my_pending != 0)) {
        // the exact maximum over the candidates, then the undecided blocks
        // against the exact threshold
        double m = -DBL_MAX;
        uint32_t any = __ballot_sync(0xffffffffu, my_cand != 0);
        while (any) {
            const int w = __ffs(any) - 1;
            any &= any - 1;
            uint32_t cb = __shfl_sync(0xffffffffu, my_cand, w);
            while (cb) {
                const int l = __ffs(cb) - 1;
                cb &= cb - 1;
                m = fmax(m, score64<HD>(q64, W.kbar64 + ((int64_t)(b0 + 32 * w + l) * D.Hkv + g) * HD, D.G));
            }
        }
        const double t = D.tau * m;
        any = __ballot_sync(0xffffffffu, my_pending != 0);
        while (any) {
            const int w = __ffs(any) - 1;
            any &= any - 1;
            uint32_t pb = __shfl_sync(0xffffffffu, my_pending, w);
            while (pb) {
                const int l = __ffs(pb) - 1;
                pb &= pb - 1;
                const double x64 = score64<HD>(q64, W.kbar64 + ((int64_t)(b0 + 32 * w + l) * D.Hkv + g) * HD, D.G);
                if (lane == w && x64 >= t) my_keep |= 1u << l;
            }
        }
    }
    if (32 * lane <= i) mask[lane] = my_keep;
    count += __reduce_add_sync(0xffffffffu, __popc(my_keep));
    for (int w = i / 32 + 1 + lane; w < D.mask_words; w += 32) mask[w] = 0u;
}

// The decision of row r (warp-collective): writes its kept-mask words and
// returns its kept count.
template <int HD, bool CHUNK>
__device__ __forceinline__ int thr_row(const Dims& D, const PlanPtrs& P, const WsPtrs& W, int64_t r,
                                       int lane, bool have_bounds) {
    const int g = (int)(r / D.NB);
    const int64_t bi = r % D.NB;
    const int s = P.block_seq[bi];
    const int b0 = P.cu_blocks[s];
    const int i = (int)(bi - b0);
    uint32_t* mask = P.kept_mask + r * D.mask_words;
    int count = 0;
    if (CHUNK && i < P.q_off[s] / D.B) {
        // query block below a chunk: no row, nothing kept
        for (int w = lane; w < D.mask_words; w += 32) mask[w] = 0u;
    } else if (D.tau == 0.0) {
        for (int w = lane; w < D.mask_words; w += 32) {
            uint32_t bits = 0;
            if (32 * w + 31 <= i) bits = 0xFFFFFFFFu;
            else if (32 * w <= i) bits = (1u << (i - 32 * w + 1)) - 1u;
            mask[w] = bits;
        }
        count = i + 1;
    } else {
        const float* sc = W.scores + (int64_t)g * D.tri_total + P.tri_off[s] + (int64_t)i * (i + 1) / 2;
        const double inv_sqrt_d = 1.0 / sqrt((double)HD);
        const double qr = W.qres[bi * D.Hkv + g];
        RowBound rb;
        rb.kb = W.kb2 + (int64_t)g * D.NB + b0;   // contiguous in j
        // (1 + 2^-20: far above the float64 rounding of the tests below)
        rb.A = qr * inv_sqrt_d * (1.0 + 0x1p-20);
        rb.B = ((double)W.qnorm[bi * D.Hkv + g] + qr) * inv_sqrt_d * (1.0 + 0x1p-20);
        if (have_bounds && i < 32 * 32) {
            thr_one_pass<HD>(D, W, sc, rb, W.bounds[2 * r], W.bounds[2 * r + 1], i, bi, b0, g, lane, mask,
                             count);
        } else {
            // largest lower bound of any score (kThrBatch words of loads at a time)
            double m_lo = -DBL_MAX;
#pragma unroll 1
            for (int jb = 0; jb <= i; jb += 32 * kThrBatch) {
                float xs[kThrBatch], ks[kThrBatch], rs[kThrBatch];
#pragma unroll
                for (int u = 0; u < kThrBatch; ++u) {
                    const int j = jb + 32 * u + lane;
                    xs[u] = j <= i ? __ldg(sc + j) : 0.f;
                    const float2 t2 = j <= i ? __ldg(rb.kb + j) : make_float2(0.f, 0.f);
                    ks[u] = t2.x;
                    rs[u] = t2.y;
                }
#pragma unroll
                for (int u = 0; u < kThrBatch; ++u)
                    if (jb + 32 * u + lane <= i) m_lo = fmax(m_lo, (double)xs[u] - rb.e(ks[u], rs[u]));
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m_lo = fmax(m_lo, __shfl_xor_sync(0xffffffffu, m_lo, o));
            thr_decide<HD>(D, W, sc, rb, m_lo, i, bi, b0, g, lane, mask, count);
        }
    }
    return count;
}

// Position o of the rows in the order "longest first" (block index from the
// last down, every kv-head of a block together) that warp gw of nw takes as
// its t-th row: passes of nw rows, odd passes from the other end, so that
// every warp gets rows of about the same total length.
__device__ __forceinline__ int64_t row_order(int64_t t, int64_t gw, int64_t nw) {
    return t * nw + ((t & 1) ? nw - 1 - gw : gw);
}

// The threshold: each warp takes the next item from a counter: first the
// e4m3 means' chunk maxima of one block (NB short items), then the rows
// "longest first" (their costs depend on how many blocks need re-scoring, so
// they are handed out as warps free up).  A row's decision leaves its kept
// count, added to the counts of the row's segment (kCsrRows rows) and
// super-segment (kCsrSup rows); k_csr turns the counts into offsets and
// writes the column ids.
template <int HD, bool CHUNK>
__global__ void __launch_bounds__(kThrRows * 32, 2) k_threshold(Dims D, PlanPtrs P, WsPtrs W,
                                                             bool have_bounds) {
    // launched as a programmatic dependent: everything before it is complete
    // once the wait returns
    asm volatile("griddepcontrol.wait;" ::: "memory");
    // k_csr may be launched now: it waits for this kernel to complete
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (!*P.meta_valid) return;
    const int lane = threadIdx.x & 31;
    for (;;) {
        int o = 0;
        if (lane == 0) o = atomicAdd(P.thr_next, 1);
        o = __shfl_sync(0xffffffffu, o, 0);
        if (o < D.NB) {   // the first NB items: the e4m3 means' chunk maxima
            means_absmax(D, P, o, lane);
            continue;
        }
        o -= (int)D.NB;
        if (o >= D.R) break;
        const int64_t bi = D.NB - 1 - o / D.Hkv;
        const int64_t r = (int64_t)(o % D.Hkv) * D.NB + bi;
        const int count = thr_row<HD, CHUNK>(D, P, W, r, lane, have_bounds);
        if (lane == 0) {
            P.csr_count[r] = count;
            atomicAdd(P.csr_seg + r / kCsrRows, count);
            atomicAdd(P.csr_sup + r / kCsrSup, count);
        }
    }
}

// The CSR from the kept counts and mask words, and before the rows the e4m3
// means' codes (one item per block: their dependent loads then overlap the
// rows instead of forming the kernel's tail).  The warps take the items in row_order
// (which evens out their work); a row's offset is the kept count of every
// row before it:
// the super-segments before its own, the segments before it within its
// super-segment, and the rows before it within its segment (at most
// R / kCsrSup + 62 counts, added up by the warp's lanes).  Then the warp
// writes the row pointer and the row's column ids, ascending.  No warp waits
// on another.
__global__ void __launch_bounds__(kThrRows * 32) k_csr(Dims D, PlanPtrs P) {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (!*P.meta_valid) return;
    const int lane = threadIdx.x & 31;
    const int64_t nw = (int64_t)gridDim.x * (blockDim.x >> 5);
    const int64_t gw = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    for (int64_t t = 0; ; ++t) {
        int64_t o = row_order(t, gw, nw);
        if (o >= D.R + D.NB) break;
        if (o < D.NB) {   // first: the e4m3 means' codes of one block
            means_codes(D, P, o, lane);
            continue;
        }
        o -= D.NB;
        const int64_t bi = D.NB - 1 - o / D.Hkv;
        const int64_t r = (o % D.Hkv) * D.NB + bi;
        const int64_t seg = r / kCsrRows, sup = r / kCsrSup;
        long long part = 0;
        for (int64_t q = lane; q < sup; q += 32) part += P.csr_sup[q];
        {
            const int64_t q = sup * (kCsrSup / kCsrRows) + lane;
            if (q < seg) part += P.csr_seg[q];
            const int64_t q2 = seg * kCsrRows + lane;
            if (q2 < r) part += P.csr_count[q2];
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
        const long long base = part;
        const int count = P.csr_count[r];
        if (lane == 0) P.row_ptr[r] = (int32_t)base;
        if (r == D.R - 1 && lane == 0) P.row_ptr[D.R] = (int32_t)(base + count);
        if (count == 0) continue;
        const int i = (int)(bi - P.cu_blocks[P.block_seq[bi]]);
        const uint32_t* mask = P.kept_mask + r * D.mask_words;
        // 32 mask words at a time: lane l loads word w0 + l, the lanes' exclusive
        // sums of the words' bit counts place each word's ids
        // (positions fit in 32 bits: nnz_cap < 2^31)
        int32_t* dst = P.col_idx + base;
        const uint32_t below = (1u << lane) - 1u;
        for (int w0 = 0; 32 * w0 <= i; w0 += 32) {
            const int w = w0 + lane;
            const uint32_t bits = 32 * w <= i ? mask[w] : 0u;
            const int c = __popc(bits);
            int incl = c;
#pragma unroll
            for (int o2 = 1; o2 < 32; o2 <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incl, o2);
                if (lane >= o2) incl += y;
            }
            const int ex = incl - c;
            const int nwd = min(32, i / 32 + 1 - w0);
            int id = 32 * w0 + lane;
            for (int u = 0; u < nwd; ++u, id += 32) {
                const uint32_t b = __shfl_sync(0xffffffffu, bits, u);
                const int a = __shfl_sync(0xffffffffu, ex, u) + __popc(b & below);
                if (((b >> lane) & 1u) && FP2_CHECK(base + a < D.nnz_cap, P.status)) dst[a] = id;
            }
            dst += __shfl_sync(0xffffffffu, incl, 31);
        }
    }
}

// Launch with programmatic stream serialization: the kernel may begin before
// the one before it in the stream completes; what it may read before its
// griddepcontrol.wait is stated at each kernel.
template <typename... KArgs, typename... Args>
int launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
               Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, args...) == cudaSuccess ? FP2_OK : FP2_ERR_CUDA;
}

template <int HD, int GQ>
int launch_score_pipe(const Dims& D, const PlanPtrs& P, const WsPtrs& W, const CUtensorMap& tq,
                      const CUtensorMap& tk, int grid, cudaStream_t st) {
    const int smem = ScorePCfg<HD>::kSmem;
    if (cudaFuncSetAttribute(k_score_pipe<HD, GQ>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
        cudaSuccess)
        return FP2_ERR_CUDA;
    return launch_pdl(k_score_pipe<HD, GQ>, dim3(grid), dim3(kScorePThreads), (size_t)smem, st, D, P, W,
                      tq, tk);
}

// Scores (tau > 0), the threshold and the CSR.
template <int HD>
int launch_score(const Dims& D, const PlanPtrs& P, const WsPtrs& W, cudaStream_t st) {
    if (D.tau > 0.0) {
        // tensor maps over the tf32-rounded query and key block means
        CUtensorMap tq, tk;
        const uint64_t qd[3] = {(uint64_t)HD, (uint64_t)D.Hq, (uint64_t)D.NB};
        const uint64_t qs[2] = {(uint64_t)HD * 4, (uint64_t)D.Hq * HD * 4};
        const uint32_t qb[3] = {32u, (uint32_t)D.G, (uint32_t)D.rows_per_group};
        const uint64_t kd[3] = {(uint64_t)HD, (uint64_t)D.Hkv, (uint64_t)D.NB};
        const uint64_t ks[2] = {(uint64_t)HD * 4, (uint64_t)D.Hkv * HD * 4};
        const uint32_t kb[3] = {32u, 1u, (uint32_t)kScoreKeys};
        if (!make_tensor_map(&tq, W.qbar32, 3, qd, qs, qb, kMapF32) ||
            !make_tensor_map(&tk, W.kbar_tf, 3, kd, ks, kb, kMapF32))
            return FP2_ERR_CUDA;
        int rc;
        if (D.G <= 32 && (D.G & (D.G - 1)) == 0) {
            // the G heads of a block are G aligned, adjacent lanes of one warp
            const int64_t items = (int64_t)D.n_groups_cap * D.Hkv;
            const int grid = (int)std::min<int64_t>(items, std::max(1, sm_count()));
            switch (D.G) {
                case 1: rc = launch_score_pipe<HD, 1>(D, P, W, tq, tk, grid, st); break;
                case 2: rc = launch_score_pipe<HD, 2>(D, P, W, tq, tk, grid, st); break;
                case 4: rc = launch_score_pipe<HD, 4>(D, P, W, tq, tk, grid, st); break;
                case 8: rc = launch_score_pipe<HD, 8>(D, P, W, tq, tk, grid, st); break;
                case 16: rc = launch_score_pipe<HD, 16>(D, P, W, tq, tk, grid, st); break;
                default: rc = launch_score_pipe<HD, 32>(D, P, W, tq, tk, grid, st); break;
            }
        } else {
            const int smem = ScoreTcCfg<HD>::kSmem;
            if (cudaFuncSetAttribute(k_score_tc<HD>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     smem) != cudaSuccess)
                return FP2_ERR_CUDA;
            const int64_t items = D.score_tiles * D.Hkv;
            const int grid = (int)std::min<int64_t>(items, std::max(1, sm_count()));
            rc = launch_pdl(k_score_tc<HD>, dim3(grid), dim3(kScoreTcThreads), smem, st, D, P, W, tq, tk);
        }
        if (rc != FP2_OK) return rc;
    }
    // the pipelined scorer leaves each row's score bounds for the threshold
    const bool bounds = D.tau > 0.0 && D.G <= 32 && (D.G & (D.G - 1)) == 0;
    // the threshold's CTAs take rows until none is left: as many CTAs as fit
    // on the device at once
    auto thr = P.cu_q ? k_threshold<HD, true> : k_threshold<HD, false>;
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, thr, kThrRows * 32, 0) != cudaSuccess)
        return FP2_ERR_CUDA;
    const int64_t fit = (int64_t)std::max(1, per_sm) * std::max(1, sm_count());
    const int64_t need = (D.R + D.NB + kThrRows - 1) / kThrRows;
    const dim3 grid((unsigned)std::min(fit, need));
    int rc = launch_pdl(thr, grid, dim3(kThrRows * 32), 0, st, D, P, W, bounds);
    if (rc != FP2_OK) return rc;
    int csr_per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&csr_per_sm, k_csr, kThrRows * 32, 0) != cudaSuccess)
        return FP2_ERR_CUDA;
    const int64_t csr_fit = (int64_t)std::max(1, csr_per_sm) * std::max(1, sm_count());
    return launch_pdl(k_csr, dim3((unsigned)std::min(csr_fit, need)), dim3(kThrRows * 32), 0, st, D, P);
}

}  // namespace

namespace {

template <bool KV8, bool CHUNK, bool BYVAL, bool NORMS>
void launch_pool(const Layout& L, const fp2_problem* p, const SeqMap& M, const void* q,
                 const void* k, const void* v, const float* k_scale, const float* v_scale,
                 const PlanPtrs& P, const WsPtrs& W, cudaStream_t st) {
    const Dims& D = L.dims;
    const int vecs = (D.Hq + 2 * D.Hkv) * D.d / 8;
    dim3 grid((unsigned)D.NB, (vecs + kPoolThreads - 1) / kPoolThreads);
    k_pool<KV8, CHUNK, BYVAL, NORMS><<<grid, kPoolThreads, 0, st>>>(
        D, M, L.Tq, p->cu_seqlens, p->page_table, static_cast<const uint16_t*>(q), k, v, k_scale,
        v_scale, CHUNK ? p->prev_kbar : nullptr, CHUNK ? p->prev_vbar : nullptr, P, W);
}

template <bool KV8, bool CHUNK>
void launch_pool_kv(const Layout& L, const fp2_problem* p, const SeqMap& M, bool byval, bool norms,
                    const void* q, const void* k, const void* v, const float* ks, const float* vs,
                    const PlanPtrs& P, const WsPtrs& W, cudaStream_t st) {
    if (byval) {
        if (norms) launch_pool<KV8, CHUNK, true, true>(L, p, M, q, k, v, ks, vs, P, W, st);
        else launch_pool<KV8, CHUNK, true, false>(L, p, M, q, k, v, ks, vs, P, W, st);
    } else {
        if (norms) launch_pool<KV8, CHUNK, false, true>(L, p, M, q, k, v, ks, vs, P, W, st);
        else launch_pool<KV8, CHUNK, false, false>(L, p, M, q, k, v, ks, vs, P, W, st);
    }
}

}  // namespace

int launch_plan(const Layout& L, const fp2_problem* p, const void* q, const void* k, const void* v,
                const PlanPtrs& P0, const WsPtrs& W, cudaStream_t st, const float* k_scale,
                const float* v_scale) {
    const Dims& D = L.dims;
    PlanPtrs P = P0;
    P.cu_q = L.chunked ? p->cu_q_seqlens : nullptr;
    // The pooling kernel runs first when the sequences fit the by-value map:
    // it then needs nothing from k_meta, which is launched after it as a
    // programmatic dependent (it may start once every pooling CTA has begun,
    // overlapping the pool's last wave) and waits for it before completing.
    const bool byval = D.n_seqs <= kMapSeqs;
    SeqMap M;
    std::memset(&M, 0, sizeof(M));
    if (byval) {
        M.n = D.n_seqs;
        for (int s = 0; s < D.n_seqs; ++s) {
            const int Ls = p->seqlens[s];
            const int Qs = L.chunked ? p->q_seqlens[s] : Ls;
            M.cu_blocks[s + 1] = M.cu_blocks[s] + (Ls + D.B - 1) / D.B;
            M.cu_tok[s + 1] = M.cu_tok[s] + Ls;
            M.cu_q[s + 1] = M.cu_q[s] + Qs;
            M.q_off[s] = Ls - Qs;
        }
    }
    // the threshold's error-bound norms come out of the pooling kernel when
    // the G query heads of a kv-head fall into one pooling CTA (1024 columns)
    const bool norms_in_pool = D.tau > 0.0 && (kPoolThreads * 8) % (D.G * D.d) == 0;
    auto meta = [&]() -> int {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(1);
        cfg.blockDim = dim3(kMetaThreads);
        cfg.dynamicSmemBytes = 0;
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = byval ? 1 : 0;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        return cudaLaunchKernelEx(&cfg, k_meta, D, L.sched, p->cu_seqlens, p->page_table, L.Tq, P) ==
                       cudaSuccess
                   ? FP2_OK
                   : FP2_ERR_CUDA;
    };
    auto pool = [&]() {
        if (k_scale)   // (an FP8 KV cache is never chunked: the entry point rejects it)
            launch_pool_kv<true, false>(L, p, M, byval, norms_in_pool, q, k, v, k_scale, v_scale, P, W, st);
        else if (L.chunked)
            launch_pool_kv<false, true>(L, p, M, byval, norms_in_pool, q, k, v, nullptr, nullptr, P, W, st);
        else
            launch_pool_kv<false, false>(L, p, M, byval, norms_in_pool, q, k, v, nullptr, nullptr, P, W, st);
    };
    if (byval) {
        pool();
        if (meta() != FP2_OK) return FP2_ERR_CUDA;
    } else {
        if (meta() != FP2_OK) return FP2_ERR_CUDA;
        pool();
    }
    if (D.tau > 0.0 && !norms_in_pool) {
        const int64_t warps = D.NB * D.Hkv;
        k_norms<<<(unsigned)((warps * 32 + 255) / 256), 256, 0, st>>>(D, P, W);
    }
    int rc = D.d == 64 ? launch_score<64>(D, P, W, st) : launch_score<128>(D, P, W, st);
    if (rc != FP2_OK) return rc;
    return cudaGetLastError() == cudaSuccess ? FP2_OK : FP2_ERR_CUDA;
}

}  // namespace fp2
