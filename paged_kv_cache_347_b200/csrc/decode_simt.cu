// CUDA-core paged decode and the split-partial reduce.
//
// Attention over the block table (mbrenndoerfer.com "Paged Attention >
// Summary", bullet 3: K/V read through the table one block at a time with an
// online softmax, no gather into a contiguous buffer).  This kernel serves the
// fp32 cache (where the output must match to 1e-5, so the dot products stay
// in fp32 FMA), block size 4, and any shape the tensor-core kernel does not
// take.
//
// Work unit: one CTA per (split, KV head g, sequence s) walks the tokens of
// its split.  A "token group" of D/E lanes (E = elements per 16-byte word)
// holds one K row -- every lane loads one 16-byte word, so a group reads a
// whole row with one coalesced transaction -- and keeps its slice of q for
// all G query heads of the KV head, so each K/V row is read once for the
// whole GQA group.  A warp takes 32/(D/E) tokens per step; the online-softmax
// running max is warp-uniform per head and the running sums and outputs are
// per lane, merged over the warp and then over the CTA's warps at the end.
#include <math.h>

#include "decode_common.cuh"

namespace pa {

constexpr int kSimtThreads = 128;

template <typename T, int D, int GM>
__global__ void __launch_bounds__(kSimtThreads) decode_simt_kernel(DecodeParams p) {
    constexpr int E = Vec16<T>::N;  // elements per 16-byte word
    constexpr int TG = D / E;       // lanes per token
    constexpr int TPW = 32 / TG;    // tokens per warp step
    constexpr int NW = kSimtThreads / 32;
    static_assert(TG <= 32 && 32 % TG == 0, "head_dim / vector width");

    __shared__ float sm_o[NW][GM][D + 4];
    __shared__ float sm_m[NW][GM];
    __shared__ float sm_l[NW][GM];

    const int split = blockIdx.x, g = blockIdx.y, s = blockIdx.z;
    const int L = checked_seq_len(p, s, split == 0 && g == 0 && threadIdx.x == 0);
    const int nsplit = num_splits_for(L, p.partition_size);
    if (split >= nsplit) return;

    const int G = p.num_heads / p.num_kv_heads;
    const int Hkv = p.num_kv_heads;
    const int bs = p.block_size;
    const int t0 = split * p.partition_size;
    const int t1 = min(L, t0 + p.partition_size);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int slot = lane / TG, li = lane % TG;

    const T *qp = static_cast<const T *>(p.q) + ((int64_t)s * p.num_heads + g * G) * D + li * E;
    float qf[GM][E];
#pragma unroll
    for (int h = 0; h < GM; ++h) {
        if (h < G) {
            Vec16<T>::unpack(*reinterpret_cast<const uint4 *>(qp + h * D), qf[h]);
        } else {
#pragma unroll
            for (int e = 0; e < E; ++e) qf[h][e] = 0.f;
        }
    }

    const T *kc = static_cast<const T *>(p.k_cache);
    const T *vc = static_cast<const T *>(p.v_cache);
    float m[GM], l[GM], o[GM][E];
#pragma unroll
    for (int h = 0; h < GM; ++h) {
        m[h] = -INFINITY;
        l[h] = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) o[h][e] = 0.f;
    }

    for (int base = t0 + warp * TPW; base < t1; base += NW * TPW) {
        const int t = base + slot;
        const bool valid = t < t1;
        float kf[E], vf[E];
#pragma unroll
        for (int e = 0; e < E; ++e) kf[e] = vf[e] = 0.f;
        if (valid) {
            const int pb = checked_block(p, s, t / bs);
            if (pb >= 0) {
                const int64_t row = ((int64_t)pb * Hkv + g) * bs + t % bs;
                const uint4 ku = __ldg(reinterpret_cast<const uint4 *>(kc + row * D + li * E));
                const uint4 vu = __ldg(reinterpret_cast<const uint4 *>(vc + row * D + li * E));
                Vec16<T>::unpack(ku, kf);
                Vec16<T>::unpack(vu, vf);
            }
        }
#pragma unroll
        for (int h = 0; h < GM; ++h) {
            float acc = 0.f;
#pragma unroll
            for (int e = 0; e < E; ++e) acc = fmaf(qf[h][e], kf[e], acc);
#pragma unroll
            for (int off = TG / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
            const float x = valid ? acc * p.scale_log2 : -INFINITY;
            float cm = x;
#pragma unroll
            for (int off = TG; off < 32; off <<= 1) cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, off));
            const float mn = fmaxf(m[h], cm);  // finite: slot 0 of every step is valid
            const float al = exp2f(m[h] - mn);
            const float pr = exp2f(x - mn);
            l[h] = l[h] * al + pr;
#pragma unroll
            for (int e = 0; e < E; ++e) o[h][e] = fmaf(pr, vf[e], o[h][e] * al);
            m[h] = mn;
        }
    }

    // sums over the warp's token slots
#pragma unroll
    for (int h = 0; h < GM; ++h) {
#pragma unroll
        for (int off = TG; off < 32; off <<= 1) {
            l[h] += __shfl_xor_sync(0xffffffffu, l[h], off);
#pragma unroll
            for (int e = 0; e < E; ++e) o[h][e] += __shfl_xor_sync(0xffffffffu, o[h][e], off);
        }
    }
    if (slot == 0) {
#pragma unroll
        for (int h = 0; h < GM; ++h) {
#pragma unroll
            for (int e = 0; e < E; ++e) sm_o[warp][h][li * E + e] = o[h][e];
        }
    }
    if (lane == 0) {
#pragma unroll
        for (int h = 0; h < GM; ++h) {
            sm_m[warp][h] = m[h];
            sm_l[warp][h] = l[h];
        }
    }
    __syncthreads();

    // merge the warps: out = sum_w 2^(m_w - M) o_w / sum_w 2^(m_w - M) l_w
    for (int idx = threadIdx.x; idx < G * D; idx += kSimtThreads) {
        const int h = idx / D, d = idx - (idx / D) * D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < NW; ++w) M = fmaxf(M, sm_m[w][h]);
        float num = 0.f, den = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < NW; ++w) {
                const float sc = exp2f(sm_m[w][h] - M);
                num = fmaf(sc, sm_o[w][h][d], num);
                den = fmaf(sc, sm_l[w][h], den);
            }
        }
        store_unit(p, s, g * G + h, split, nsplit, d, M, den, num);
    }
}

// Merge of the split partials: one CTA per (query head, sequence) with more
// than one split.  out = sum_x 2^(m_x - M) o_x / sum_x 2^(m_x - M) l_x with
// M = max_x m_x (m in log2 units).  The partials were just written by the main
// kernel and are read from L2; the CTA's threads split the splits between
// them (kReduceThreads / D groups) so many loads are in flight at once.
constexpr int kReduceThreads = 256;

__global__ void __launch_bounds__(kReduceThreads) decode_reduce_kernel(DecodeParams p) {
    // launched as a programmatic dependent of the main kernel: wait for its
    // partials to be complete and visible
    pdl_wait_prior_grid();
    const int h = blockIdx.x, s = blockIdx.y;
    const int L = checked_seq_len(p, s, false);
    const int nsplit = num_splits_for(L, p.partition_size);
    if (nsplit <= 1) return;
    __shared__ float red[kReduceThreads / 32];
    __shared__ float part[kReduceThreads];
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int64_t u0 = ((int64_t)s * p.num_heads + h) * p.max_splits;
    const float *ml = p.part_ml + 2 * u0;

    float M = -INFINITY;
    for (int x = tid; x < nsplit; x += kReduceThreads) M = fmaxf(M, __ldg(ml + 2 * x));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    if (lane == 0) red[wid] = M;
    __syncthreads();
    M = red[0];
#pragma unroll
    for (int w = 1; w < kReduceThreads / 32; ++w) M = fmaxf(M, red[w]);
    __syncthreads();

    float den = 0.f;
    for (int x = tid; x < nsplit; x += kReduceThreads)
        den = fmaf(exp2f(__ldg(ml + 2 * x) - M), __ldg(ml + 2 * x + 1), den);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) den += __shfl_xor_sync(0xffffffffu, den, off);
    if (lane == 0) red[wid] = den;

    const int D = p.head_dim;
    const int groups = kReduceThreads / D;
    const int grp = tid / D, d = tid - grp * D;
    const float *po = p.part_o + u0 * D + d;
    float num = 0.f;
    int x = grp;
    for (; x + 3 * groups < nsplit; x += 4 * groups) {
        const float w0 = exp2f(__ldg(ml + 2 * x) - M);
        const float w1 = exp2f(__ldg(ml + 2 * (x + groups)) - M);
        const float w2 = exp2f(__ldg(ml + 2 * (x + 2 * groups)) - M);
        const float w3 = exp2f(__ldg(ml + 2 * (x + 3 * groups)) - M);
        const float a0 = __ldg(po + (int64_t)x * D);
        const float a1 = __ldg(po + (int64_t)(x + groups) * D);
        const float a2 = __ldg(po + (int64_t)(x + 2 * groups) * D);
        const float a3 = __ldg(po + (int64_t)(x + 3 * groups) * D);
        num = fmaf(w0, a0, fmaf(w1, a1, fmaf(w2, a2, fmaf(w3, a3, num))));
    }
    for (; x < nsplit; x += groups) num = fmaf(exp2f(__ldg(ml + 2 * x) - M), __ldg(po + (int64_t)x * D), num);
    part[tid] = num;
    __syncthreads();
    if (tid < D) {
        float tot = 0.f;
        for (int gq = 0; gq < groups; ++gq) tot += part[gq * D + tid];
        float dsum = 0.f;
#pragma unroll
        for (int w = 0; w < kReduceThreads / 32; ++w) dsum += red[w];
        p.out[((int64_t)s * p.num_heads + h) * D + tid] = dsum > 0.f ? tot / dsum : 0.f;
    }
}

template <typename T, int D>
static cudaError_t launch_simt_d(const DecodeParams &p, cudaStream_t stream) {
    const dim3 grid(p.max_splits, p.num_kv_heads, p.num_seqs);
    const int G = p.num_heads / p.num_kv_heads;
    if (G <= 1)
        decode_simt_kernel<T, D, 1><<<grid, kSimtThreads, 0, stream>>>(p);
    else if (G <= 2)
        decode_simt_kernel<T, D, 2><<<grid, kSimtThreads, 0, stream>>>(p);
    else if (G <= 4)
        decode_simt_kernel<T, D, 4><<<grid, kSimtThreads, 0, stream>>>(p);
    else
        decode_simt_kernel<T, D, 8><<<grid, kSimtThreads, 0, stream>>>(p);
    return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_simt_t(const DecodeParams &p, cudaStream_t stream) {
    return p.head_dim == 64 ? launch_simt_d<T, 64>(p, stream) : launch_simt_d<T, 128>(p, stream);
}

cudaError_t launch_decode_simt(const DecodeParams &p, int dtype, cudaStream_t stream) {
    if (p.num_seqs == 0) return cudaSuccess;
    switch (dtype) {
    case PA_F32: return launch_simt_t<float>(p, stream);
    case PA_BF16: return launch_simt_t<__nv_bfloat16>(p, stream);
    case PA_F16: return launch_simt_t<__half>(p, stream);
    default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_decode_reduce(const DecodeParams &p, cudaStream_t stream) {
    if (p.max_splits <= 1 || p.num_seqs == 0) return cudaSuccess;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.num_heads, p.num_seqs);
    cfg.blockDim = dim3(kReduceThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_reduce_kernel, p);
}

}  // namespace pa
