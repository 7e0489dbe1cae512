// Direct online FP8 quantisation (Table 1 footnote of the metallab.ai
// summary of arXiv 2608.19758: "direct online FP8 quantization"): one CTA
// per (block, head) finds the absmax of the block's bf16 values, sets
// scale = absmax / 448 (1 for an all-zero block) and writes
// e4m3 = round-to-nearest-even-saturating(x / scale), with scale and quotient
// in fp32.  For a chunked problem a query block covers the chunk's positions
// in it (a block below the chunk gets scale 1 and no codes).  Memory bound: the block is read twice (the second pass mostly
// from L2) and written once at a quarter of the size.
#include "fp2_device.cuh"

namespace fp2 {

namespace {

constexpr int kQuantThreads = 128;

// Two floats -> packed e4m3x2 (lo in the low byte), RNE, saturating.
__device__ __forceinline__ uint16_t pack_e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// Address (in elements) of token t of sequence s, head h, element e.
struct Addr {
    const Dims* D;
    const int32_t* cu_seqlens;
    const int32_t* page_table;
    bool paged;
    int H;      // heads per token of the tensor (all of a layer's heads for a slice)
    int pos0;   // position of the sequence's first row (a chunk's first query)
    __device__ __forceinline__ int64_t operator()(int s, int t, int h, int e) const {
        if (!paged) return ((int64_t)(cu_seqlens[s] + t - pos0) * H + h) * D->d + e;
        const int id = page_table[(int64_t)s * D->pt_stride + t / 64];
        if (id < 0 || id >= D->num_pages) return -1;
        return (((int64_t)id * 64 + t % 64) * H + h) * D->d + e;
    }
};

// The tensors of one launch: q, k and v with their codes and scales (a
// single-tensor launch fills only `which`).
struct QuantArgs {
    const uint16_t* x[3];
    uint8_t* x8[3];
    float* scales[3];
};

// One CTA per (block, head): blockIdx.y runs over the heads of the tensors
// the launch quantises, q's Hq heads first, then k's and v's Hkv heads.
__global__ void __launch_bounds__(kQuantThreads)
k_quant(Dims D, const int32_t* __restrict__ cu_seqlens, const int32_t* __restrict__ page_table,
        PlanPtrs P, QuantArgs A, int first) {
    if (!*P.meta_valid) return;
    const int64_t b = blockIdx.x;
    int which = first, h = blockIdx.y;
    while (h >= (which == 0 ? D.Hq : D.Hkv)) {
        h -= which == 0 ? D.Hq : D.Hkv;
        ++which;
    }
    const uint16_t* __restrict__ x = A.x[which];
    uint8_t* __restrict__ x8 = A.x8[which];
    float* __restrict__ scales = A.scales[which];
    const int H = which == 0 ? D.Hq : D.Hkv;
    const int s = P.block_seq[b];
    const int i = (int)(b - P.cu_blocks[s]);
    const int L = cu_seqlens[s + 1] - cu_seqlens[s];
    int t0 = i * D.B;
    const int t1 = min(t0 + D.B, L);
    // q of a chunked problem holds positions q_off .. L - 1 of each sequence:
    // a query block's scale covers its chunk positions (none below the chunk)
    const int32_t* base = cu_seqlens;
    int pos0 = 0;
    if (which == 0 && P.cu_q) {
        t0 = max(t0, P.q_off[s]);
        base = P.cu_q;
        pos0 = P.q_off[s];
    }
    Addr addr{&D, base, page_table, which != 0 && D.page_size != 0,
              which == 0 ? D.Hq_str : D.Hkv_str, pos0};
    const int vpt = D.d / 8;                       // 16-byte vectors per token
    const int nvec = t1 > t0 ? (t1 - t0) * vpt : 0;

    float amax = 0.f;
    for (int idx = threadIdx.x; idx < nvec; idx += kQuantThreads) {
        const int t = t0 + idx / vpt, e = (idx % vpt) * 8;
        const int64_t a = addr(s, t, h, e);
        if (a < 0) continue;
        const uint4 v = *reinterpret_cast<const uint4*>(x + a);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            amax = fmaxf(amax, fabsf(__uint_as_float(w[k] << 16)));
            amax = fmaxf(amax, fabsf(__uint_as_float(w[k] & 0xFFFF0000u)));
        }
    }
    __shared__ float red[kQuantThreads / 32];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
    __syncthreads();
    amax = red[0];
    for (int k = 1; k < kQuantThreads / 32; ++k) amax = fmaxf(amax, red[k]);
    const float scale = amax > 0.f ? __fdiv_rn(amax, 448.0f) : 1.0f;
    if (threadIdx.x == 0) scales[b * H + h] = scale;

    for (int idx = threadIdx.x; idx < nvec; idx += kQuantThreads) {
        const int t = t0 + idx / vpt, e = (idx % vpt) * 8;
        const int64_t a = addr(s, t, h, e);
        if (a < 0) continue;
        const uint4 v = *reinterpret_cast<const uint4*>(x + a);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        uint32_t out[2];
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const float f0 = __fdiv_rn(__uint_as_float(w[2 * k] << 16), scale);
            const float f1 = __fdiv_rn(__uint_as_float(w[2 * k] & 0xFFFF0000u), scale);
            const float f2 = __fdiv_rn(__uint_as_float(w[2 * k + 1] << 16), scale);
            const float f3 = __fdiv_rn(__uint_as_float(w[2 * k + 1] & 0xFFFF0000u), scale);
            out[k] = (uint32_t)pack_e4m3x2(f0, f1) | ((uint32_t)pack_e4m3x2(f2, f3) << 16);
        }
        *reinterpret_cast<uint2*>(x8 + a) = make_uint2(out[0], out[1]);
    }
}

}  // namespace

int launch_quantize(const Layout& L, const fp2_problem* p, const PlanPtrs& pp, const void* const* x,
                    void* const* x8, float* const* scales, int first, int count, cudaStream_t st) {
    const Dims& D = L.dims;
    PlanPtrs P = pp;
    P.cu_q = L.chunked ? p->cu_q_seqlens : nullptr;
    QuantArgs A{};
    int heads = 0;
    for (int w = first; w < first + count; ++w) {
        A.x[w] = static_cast<const uint16_t*>(x[w - first]);
        A.x8[w] = static_cast<uint8_t*>(x8[w - first]);
        A.scales[w] = scales[w - first];
        heads += w == 0 ? D.Hq : D.Hkv;
    }
    dim3 grid((unsigned)D.NB, (unsigned)heads);
    k_quant<<<grid, kQuantThreads, 0, st>>>(D, p->cu_seqlens, p->page_table, P, A, first);
    return cudaGetLastError() == cudaSuccess ? FP2_OK : FP2_ERR_CUDA;
}

}  // namespace fp2
