// Stage 1 of FlashPrefill V2 ("pattern discovery", Figure 3 of the
// metallab.ai summary of arXiv 2608.19758): block-mean pooling, block
// scores under PackGQA, max-based thresholding and the CSR block index.
//
// Kernels, in launch order:
//   meta     one CTA: checks cu_seqlens, derives block / scoring-group maps.
//   pool     HBM-bound: streams Q, K, V once with 16-byte coalesced loads and
//            accumulates each block's sum in float64 (exact for bf16 inputs),
//            writing Qbar (fp64 workspace) and Kbar/Vbar (fp32, bf16, fp64).
//   norms    |Qbar|, |Kbar| per block and kv-head (for the score error bound).
//   score    per (sequence, kv-head, group of query blocks): float32 scores
//            of every visible key block, then the threshold decision per row.
//            A block whose float32 score lies within the float32 rounding
//            bound of the threshold, and every candidate for the row maximum,
//            is re-scored in float64, so the kept set is the one float64
//            scores give.
//   scan     row_ptr = exclusive prefix sum of kept counts.
//   compact  col_idx from the kept-block bit masks, ascending per row.
#include <cfloat>
#include <cmath>

#include "fp2_device.cuh"

namespace fp2 {

namespace {

// ---------------------------------------------------------------------------
// meta: sequence -> block and scoring-group maps, device-side checks
// ---------------------------------------------------------------------------

__global__ void k_meta(Dims D, const int32_t* __restrict__ cu_seqlens,
                       const int32_t* __restrict__ page_table, PlanPtrs P) {
    __shared__ int s_valid;
    if (threadIdx.x == 0) {
        int valid = cu_seqlens[0] == 0;
        int64_t nb_sum = 0, tri = 0, grp = 0;
        for (int s = 0; s < D.n_seqs && valid; ++s) {
            const int64_t L = (int64_t)cu_seqlens[s + 1] - cu_seqlens[s];
            if (L < 1) { valid = 0; break; }
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
            valid = (cu_seqlens[D.n_seqs] == D.T) && (nb_sum == D.NB) && (tri == D.tri_total);
            P.cu_blocks[D.n_seqs] = (int32_t)nb_sum;
            P.tri_off[D.n_seqs] = tri;
            P.group_cu[D.n_seqs] = (int32_t)grp;
        }
        *P.status = valid ? 0 : (int32_t)FP2_STATUS_BAD_SEQLENS;
        *P.meta_valid = valid;
        s_valid = valid;
    }
    __syncthreads();
    if (!s_valid) return;
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

__global__ void __launch_bounds__(kPoolThreads)
k_pool(Dims D, const int32_t* __restrict__ cu_seqlens, const int32_t* __restrict__ page_table,
       const uint16_t* __restrict__ q, const uint16_t* __restrict__ k,
       const uint16_t* __restrict__ v, PlanPtrs P, WsPtrs W) {
    if (!*P.meta_valid) return;
    const int vec = blockIdx.y * kPoolThreads + threadIdx.x;   // 8-element column chunk
    const int d = D.d;
    const int qcols = D.Hq * d, kvcols = D.Hkv * d;
    const int col = vec * 8;
    if (col >= qcols + 2 * kvcols) return;
    const int64_t b = blockIdx.x;
    const int s = P.block_seq[b];
    const int i = (int)(b - P.cu_blocks[s]);
    const int64_t tok0 = cu_seqlens[s];
    const int L = cu_seqlens[s + 1] - cu_seqlens[s];
    const int t_begin = i * D.B;
    const int t_end = min(t_begin + D.B, L);

    int which, head, e0;
    if (col < qcols) { which = 0; head = col / d; e0 = col % d; }
    else if (col < qcols + kvcols) { which = 1; head = (col - qcols) / d; e0 = (col - qcols) % d; }
    else { which = 2; head = (col - qcols - kvcols) / d; e0 = (col - qcols - kvcols) % d; }

    double acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.0;

    if (which == 0 || D.page_size == 0) {
        const uint16_t* base = which == 0 ? q : (which == 1 ? k : v);
        const int H = which == 0 ? D.Hq : D.Hkv;
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
        const uint16_t* pool = which == 1 ? k : v;
        const int64_t stride = (int64_t)D.Hkv * d / 8;
        for (int t = t_begin; t < t_end; t += 64) {
            const int id = page_table[(int64_t)s * D.pt_stride + t / 64];
            const int n = min(64, t_end - t);
            if (id < 0 || id >= D.num_pages) continue;   // recorded by k_meta; reads as zeros
            const uint4* p = reinterpret_cast<const uint4*>(pool + ((int64_t)id * 64 * D.Hkv + head) * d + e0);
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

    const double inv_n = 1.0 / (double)(t_end - t_begin);
    double m[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) m[e] = acc[e] * inv_n;
    if (which == 0) {
        double* dst = W.qbar64 + (b * D.Hq + head) * d + e0;
#pragma unroll
        for (int e = 0; e < 8; e += 2) *reinterpret_cast<double2*>(dst + e) = make_double2(m[e], m[e + 1]);
    } else {
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
        }
    }
}

// ---------------------------------------------------------------------------
// norms: one warp per (block, kv-head)
// ---------------------------------------------------------------------------

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

__global__ void k_norms(Dims D, PlanPtrs P, WsPtrs W) {
    if (!*P.meta_valid) return;
    const int64_t wid = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (wid >= D.NB * D.Hkv) return;
    const int64_t b = wid / D.Hkv;
    const int g = (int)(wid % D.Hkv);
    const int d = D.d;
    double kk = 0.0;
    const double* kp = W.kbar64 + (b * D.Hkv + g) * d;
    for (int e = lane; e < d; e += 32) kk += kp[e] * kp[e];
    kk = warp_sum_d(kk);
    double qmax = 0.0;
    for (int hl = 0; hl < D.G; ++hl) {
        const double* qp = W.qbar64 + (b * D.Hq + (int64_t)g * D.G + hl) * d;
        double qq = 0.0;
        for (int e = lane; e < d; e += 32) qq += qp[e] * qp[e];
        qq = warp_sum_d(qq);
        qmax = fmax(qmax, qq);
    }
    if (lane == 0) {
        W.knorm[wid] = round_up_f(sqrt(kk));
        W.qnorm[wid] = round_up_f(sqrt(qmax));
    }
}

// ---------------------------------------------------------------------------
// score: float32 scores + exact-decision thresholding
// ---------------------------------------------------------------------------

constexpr int kScoreThreads = 256;
constexpr int kScoreKC = 32;   // key blocks per chunk

template <int HD>
struct ScoreSmem {
    float q[kScoreQV][HD + 4];
    float k[kScoreKC][HD + 4];
    float dots[kScoreQV][kScoreKC + 1];
};

// float64 score of key block j for row (b_i, g): max over the group's heads.
template <int HD>
__device__ double score64(const Dims& D, const WsPtrs& W, int64_t b_i, int64_t b_j, int g) {
    const int lane = threadIdx.x & 31;
    const double* kp = W.kbar64 + (b_j * D.Hkv + g) * HD;
    double best = -DBL_MAX;
    for (int hl = 0; hl < D.G; ++hl) {
        const double* qp = W.qbar64 + (b_i * D.Hq + (int64_t)g * D.G + hl) * HD;
        double acc = 0.0;
#pragma unroll
        for (int e = lane; e < HD; e += 32) acc = fma(qp[e], kp[e], acc);
        acc = warp_sum_d(acc);
        best = fmax(best, acc);
    }
    return best / sqrt((double)HD);
}

template <int HD>
__global__ void __launch_bounds__(kScoreThreads)
k_score(Dims D, PlanPtrs P, WsPtrs W) {
    if (!*P.meta_valid) return;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    ScoreSmem<HD>& S = *reinterpret_cast<ScoreSmem<HD>*>(smem_raw);

    const int gi = blockIdx.x;
    const int g = blockIdx.y;
    const int s = P.group_seq[gi];
    if (gi >= P.group_cu[D.n_seqs]) return;
    const int RI = D.rows_per_group;
    const int G = D.G;
    const int b0 = P.cu_blocks[s];
    const int nb = P.cu_blocks[s + 1] - b0;
    const int i0 = (gi - P.group_cu[s]) * RI;
    const int i1 = min(i0 + RI, nb);
    const int nrows = i1 - i0;
    const int nqv = nrows * G;
    const int tid = threadIdx.x;
    const float inv_sqrt_d = 1.0f / sqrtf((float)HD);
    float* scores = W.scores + (int64_t)g * D.tri_total + P.tri_off[s];

    if (D.tau > 0.0) {
        // query block means of this group's rows, rounded to fp32
        for (int idx = tid; idx < kScoreQV * (HD / 4); idx += kScoreThreads) {
            const int qv = idx / (HD / 4), e = (idx % (HD / 4)) * 4;
            float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
            if (qv < nqv) {
                const int ri = qv / G, hl = qv % G;
                const double* qp = W.qbar64 + ((int64_t)(b0 + i0 + ri) * D.Hq + g * G + hl) * HD + e;
                f = make_float4((float)qp[0], (float)qp[1], (float)qp[2], (float)qp[3]);
            }
            *reinterpret_cast<float4*>(&S.q[qv][e]) = f;
        }
        const int tq = tid >> 3;   // 4 query vectors: 4*tq .. 4*tq+3
        const int tk = tid & 7;    // 4 key blocks:   4*tk .. 4*tk+3
        for (int jc = 0; jc < i1; jc += kScoreKC) {
            __syncthreads();
            for (int idx = tid; idx < kScoreKC * (HD / 4); idx += kScoreThreads) {
                const int kv = idx / (HD / 4), e = (idx % (HD / 4)) * 4;
                float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
                if (jc + kv < nb) {
                    const double* kp = W.kbar64 + ((int64_t)(b0 + jc + kv) * D.Hkv + g) * HD + e;
                    f = make_float4((float)kp[0], (float)kp[1], (float)kp[2], (float)kp[3]);
                }
                *reinterpret_cast<float4*>(&S.k[kv][e]) = f;
            }
            __syncthreads();
            float acc[4][4];
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int c = 0; c < 4; ++c) acc[a][c] = 0.f;
#pragma unroll 4
            for (int e = 0; e < HD; e += 4) {
                float4 qa[4], kb[4];
#pragma unroll
                for (int a = 0; a < 4; ++a) qa[a] = *reinterpret_cast<const float4*>(&S.q[4 * tq + a][e]);
#pragma unroll
                for (int c = 0; c < 4; ++c) kb[c] = *reinterpret_cast<const float4*>(&S.k[4 * tk + c][e]);
#pragma unroll
                for (int a = 0; a < 4; ++a)
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        acc[a][c] = fmaf(qa[a].x, kb[c].x, acc[a][c]);
                        acc[a][c] = fmaf(qa[a].y, kb[c].y, acc[a][c]);
                        acc[a][c] = fmaf(qa[a].z, kb[c].z, acc[a][c]);
                        acc[a][c] = fmaf(qa[a].w, kb[c].w, acc[a][c]);
                    }
            }
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int c = 0; c < 4; ++c) S.dots[4 * tq + a][4 * tk + c] = acc[a][c];
            __syncthreads();
            for (int idx = tid; idx < nrows * kScoreKC; idx += kScoreThreads) {
                const int ri = idx / kScoreKC, jj = idx % kScoreKC;
                const int i = i0 + ri, j = jc + jj;
                if (j <= i) {
                    float best = S.dots[ri * G][jj];
                    for (int hl = 1; hl < G; ++hl) best = fmaxf(best, S.dots[ri * G + hl][jj]);
                    scores[(int64_t)i * (i + 1) / 2 + j] = best * inv_sqrt_d;
                }
            }
        }
        __syncthreads();
    }

    // ---- per-row threshold decision: one warp per row ----
    const int warp = tid >> 5, lane = tid & 31;
    const double C = 2.0 * (HD + 8) * (1.0 / 16777216.0) / sqrt((double)HD);
    for (int ri = warp; ri < nrows; ri += kScoreThreads / 32) {
        const int i = i0 + ri;
        const int64_t bi = b0 + i;
        const int64_t r = (int64_t)g * D.NB + bi;
        uint32_t* mask = P.kept_mask + r * D.mask_words;
        int count = 0;
        if (D.tau == 0.0) {
            for (int w = lane; w < D.mask_words; w += 32) {
                uint32_t bits = 0;
                if (32 * w + 31 <= i) bits = 0xFFFFFFFFu;
                else if (32 * w <= i) bits = (1u << (i - 32 * w + 1)) - 1u;
                mask[w] = bits;
            }
            count = i + 1;
        } else {
            const float* sc = scores + (int64_t)i * (i + 1) / 2;
            const double qn = W.qnorm[bi * D.Hkv + g];
            // pass 1: largest lower bound of any score
            double m_lo = -DBL_MAX;
            for (int j = lane; j <= i; j += 32) {
                const double e = C * qn * W.knorm[(int64_t)(b0 + j) * D.Hkv + g];
                m_lo = fmax(m_lo, (double)sc[j] - e);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m_lo = fmax(m_lo, __shfl_xor_sync(0xffffffffu, m_lo, o));
            // pass 2: the row maximum in float64 over every candidate
            double m = -DBL_MAX;
            for (int jb = 0; jb <= i; jb += 32) {
                const int j = jb + lane;
                bool cand = false;
                if (j <= i) {
                    const double e = C * qn * W.knorm[(int64_t)(b0 + j) * D.Hkv + g];
                    cand = (double)sc[j] + e >= m_lo;
                }
                uint32_t cb = __ballot_sync(0xffffffffu, cand);
                while (cb) {
                    const int l = __ffs(cb) - 1;
                    cb &= cb - 1;
                    m = fmax(m, score64<HD>(D, W, bi, b0 + jb + l, g));
                }
            }
            const double t = D.tau * m;
            // pass 3: decisions (forced blocks 0 and i; uncertain ones in float64)
            for (int w = 0; 32 * w <= i; ++w) {
                const int j = 32 * w + lane;
                bool keep = false, unsure = false;
                if (j <= i) {
                    if (j == 0 || j == i) {
                        keep = true;
                    } else {
                        const double e = C * qn * W.knorm[(int64_t)(b0 + j) * D.Hkv + g];
                        const double x = (double)sc[j];
                        if (x - e >= t) keep = true;
                        else if (!(x + e < t)) unsure = true;
                    }
                }
                uint32_t ub = __ballot_sync(0xffffffffu, unsure);
                while (ub) {
                    const int l = __ffs(ub) - 1;
                    ub &= ub - 1;
                    const double x64 = score64<HD>(D, W, bi, b0 + 32 * w + l, g);
                    if (lane == l) keep = x64 >= t;
                }
                const uint32_t bits = __ballot_sync(0xffffffffu, keep);
                if (lane == 0) mask[w] = bits;
                count += __popc(bits);
            }
            for (int w = i / 32 + 1 + lane; w < D.mask_words; w += 32) mask[w] = 0u;
        }
        if (lane == 0) W.counts[r] = count;
    }
}

// ---------------------------------------------------------------------------
// scan: row_ptr = exclusive prefix sum of counts (one CTA)
// ---------------------------------------------------------------------------

constexpr int kScanThreads = 1024;

__global__ void __launch_bounds__(kScanThreads) k_scan(Dims D, PlanPtrs P, WsPtrs W) {
    if (!*P.meta_valid) return;
    __shared__ int64_t part[kScanThreads];
    const int64_t R = D.R;
    const int64_t per = (R + kScanThreads - 1) / kScanThreads;
    const int64_t lo = R < (int64_t)threadIdx.x * per ? R : (int64_t)threadIdx.x * per;
    const int64_t hi = R < lo + per ? R : lo + per;
    int64_t sum = 0;
    for (int64_t r = lo; r < hi; ++r) sum += W.counts[r];
    part[threadIdx.x] = sum;
    __syncthreads();
    for (int o = 1; o < kScanThreads; o <<= 1) {
        int64_t add = threadIdx.x >= o ? part[threadIdx.x - o] : 0;
        __syncthreads();
        part[threadIdx.x] += add;
        __syncthreads();
    }
    int64_t run = part[threadIdx.x] - sum;
    for (int64_t r = lo; r < hi; ++r) {
        P.row_ptr[r] = (int32_t)run;
        run += W.counts[r];
    }
    if (threadIdx.x == kScanThreads - 1) P.row_ptr[R] = (int32_t)part[kScanThreads - 1];
}

// ---------------------------------------------------------------------------
// compact: one warp per row writes its kept block ids in ascending order
// ---------------------------------------------------------------------------

__global__ void k_compact(Dims D, PlanPtrs P) {
    if (!*P.meta_valid) return;
    const int64_t r = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (r >= D.R) return;
    const int64_t b = r % D.NB;
    const int s = P.block_seq[b];
    const int i = (int)(b - P.cu_blocks[s]);
    const uint32_t* mask = P.kept_mask + r * D.mask_words;
    int32_t base = P.row_ptr[r];
    for (int w = 0; 32 * w <= i; ++w) {
        const uint32_t bits = mask[w];
        if ((bits >> lane) & 1u) P.col_idx[base + __popc(bits & ((1u << lane) - 1u))] = 32 * w + lane;
        base += __popc(bits);
    }
}

template <int HD>
int launch_score(const Dims& D, const PlanPtrs& P, const WsPtrs& W, cudaStream_t st) {
    const size_t smem = sizeof(ScoreSmem<HD>);
    if (cudaFuncSetAttribute(k_score<HD>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
        return FP2_ERR_CUDA;
    dim3 grid(D.n_groups_cap, D.Hkv);
    k_score<HD><<<grid, kScoreThreads, smem, st>>>(D, P, W);
    return FP2_OK;
}

}  // namespace

int launch_plan(const Layout& L, const fp2_problem* p, const void* q, const void* k, const void* v,
                const PlanPtrs& P, const WsPtrs& W, cudaStream_t st) {
    const Dims& D = L.dims;
    k_meta<<<1, 256, 0, st>>>(D, p->cu_seqlens, p->page_table, P);
    const int vecs = (D.Hq + 2 * D.Hkv) * D.d / 8;
    dim3 pool_grid((unsigned)D.NB, (vecs + kPoolThreads - 1) / kPoolThreads);
    k_pool<<<pool_grid, kPoolThreads, 0, st>>>(D, p->cu_seqlens, p->page_table,
                                               static_cast<const uint16_t*>(q),
                                               static_cast<const uint16_t*>(k),
                                               static_cast<const uint16_t*>(v), P, W);
    if (D.tau > 0.0) {
        const int64_t warps = D.NB * D.Hkv;
        k_norms<<<(unsigned)((warps * 32 + 255) / 256), 256, 0, st>>>(D, P, W);
    }
    int rc = D.d == 64 ? launch_score<64>(D, P, W, st) : launch_score<128>(D, P, W, st);
    if (rc != FP2_OK) return rc;
    k_scan<<<1, kScanThreads, 0, st>>>(D, P, W);
    k_compact<<<(unsigned)((D.R * 32 + 255) / 256), 256, 0, st>>>(D, P);
    return cudaGetLastError() == cudaSuccess ? FP2_OK : FP2_ERR_CUDA;
}

}  // namespace fp2
