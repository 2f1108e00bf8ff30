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

    const int split = blockIdx.x, g = blockIdx.y;
    const int s = seq_of(p, blockIdx.z, split == 0 && g == 0 && threadIdx.x == 0);
    if (s < 0) return;
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
    if (p.k_new != nullptr) {
        // the fused append: warp 0 of the CTA holding position L - 1 writes
        // the new token's rows; the barrier makes them visible to the L2
        // loads below
        if (warp == 0 && L > 0 && split == nsplit - 1)
            fused_append_rows(p, s, g, 1, L, (int)sizeof(T), lane);
        __syncthreads();
    }
    float m[GM], l[GM], o[GM][E];
#pragma unroll
    for (int h = 0; h < GM; ++h) {
        m[h] = -INFINITY;
        l[h] = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) o[h][e] = 0.f;
    }

    // U steps of a warp have their loads in flight together (table entry,
    // then the K and V words), then their math runs step by step
    constexpr int U = GM >= 8 ? 2 : 4;
    for (int base = t0 + warp * TPW; base < t1; base += NW * TPW * U) {
        uint4 ku[U], vu[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int t = base + u * NW * TPW + slot;
            ku[u] = vu[u] = make_uint4(0u, 0u, 0u, 0u);
            if (t < t1) {
                const int pb = checked_block(p, s, t / bs);
                if (pb >= 0) {
                    const int64_t row = ((int64_t)pb * Hkv + g) * bs + t % bs;
                    // through L2 (.cg): a row this CTA appended is read back
                    ku[u] = __ldcg(reinterpret_cast<const uint4 *>(kc + row * D + li * E));
                    vu[u] = __ldcg(reinterpret_cast<const uint4 *>(vc + row * D + li * E));
                }
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            // a step wholly past the split's end does nothing (uniform over the warp)
            if (base + u * NW * TPW >= t1) break;
            const int t = base + u * NW * TPW + slot;
            const bool valid = t < t1;
            float kf[E], vf[E];
            Vec16<T>::unpack(ku[u], kf);
            Vec16<T>::unpack(vu[u], vf);
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
    if (p.tickets != nullptr && nsplit > 1) {
        // the CTA of this (sequence, KV head) to finish last merges the splits
        __shared__ int last;
        __threadfence();
        __syncthreads();
        if (threadIdx.x == 0)
            last = ticket_arrive_last(p.tickets + (int64_t)s * p.num_kv_heads + g, p.tag, nsplit);
        __syncthreads();
        if (last) merge_splits(p, s, g * G, G, nsplit, threadIdx.x, kSimtThreads);
    }
}

// Merge of the split partials of each (sequence, query head) -- a unit:
// out = sum_x 2^(m_x - M) o_x / sum_x 2^(m_x - M) l_x with M = max_x m_x (m in
// log2 units).  The partials were just written by the main kernel and are read
// from L2, so the kernel is latency-bound: a unit takes `wpu` warps (1, 2 or
// 4, from the longest sequence's split count), each warp's lanes own 4
// consecutive d of a row (two rows per load when D = 64), and every lane
// issues the loads of up to 8 of its rows -- partial and (m, l) together --
// before it uses any, keeping a running maximum across batches of rows.  The
// warps of a unit then leave their sums in shared memory, and the last of
// them to count itself in (a shared-memory counter) combines them.
constexpr int kReduceThreads = 256;  // 8 warps
constexpr int kReduceBatch = 8;      // rows a lane has in flight

__global__ void __launch_bounds__(kReduceThreads, 4) decode_reduce_kernel(DecodeParams p, int wpu) {
    // launched as a programmatic dependent of the main kernel: wait for its
    // partials to be complete and visible
    pdl_wait_prior_grid();
    __shared__ float4 acc_s[kReduceThreads / 32][32];
    __shared__ float2 md_s[kReduceThreads / 32];
    __shared__ int arrived[kReduceThreads / 32];  // per unit (first warp's slot)
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x < kReduceThreads / 32) arrived[threadIdx.x] = 0;
    __syncthreads();
    const int64_t unit = (int64_t)blockIdx.x * (kReduceThreads / 32 / wpu) + warp / wpu;
    const int wsub = warp % wpu;
    // both exits below are taken by all the warps of a unit or by none
    if (unit >= (int64_t)p.num_seqs * p.num_heads) return;
    const int s = (int)(unit / p.num_heads);
    const int L = checked_seq_len(p, s, false);
    const int nsplit = num_splits_for(L, p.partition_size);
    if (nsplit <= 1) return;
    const int D4 = p.head_dim >> 2;  // 32 or 16
    const int rpl = 32 / D4;         // rows one warp-wide load covers: 1 or 2
    const int sub = lane / D4, c4 = lane - sub * D4;
    const int stride = wpu * rpl;    // between a lane's consecutive rows
    const int64_t u0 = unit * p.max_splits;
    const float2 *ml = reinterpret_cast<const float2 *>(p.part_ml) + u0;
    const float4 *po = reinterpret_cast<const float4 *>(p.part_o) + u0 * D4 + c4;

    float M = -INFINITY, den = 0.f;  // warp-uniform
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    // rows of this warp in a batch: x0 + sub + k * stride (k < kReduceBatch);
    // lane j < kReduceBatch * rpl loads (m, l) of row k = j / rpl, sub = j % rpl
    // and the lanes holding that row take its weight by a shuffle.  The loop
    // bound is the same for every lane of the warp (the shuffles need all).
    const int j_sub = lane % rpl, j_k = lane / rpl;
    for (int x0 = wsub * rpl; x0 < nsplit; x0 += kReduceBatch * stride) {
        float4 v_o[kReduceBatch];
#pragma unroll
        for (int k = 0; k < kReduceBatch; ++k) {
            const int x = x0 + sub + k * stride;
            v_o[k] = x < nsplit ? __ldg(po + (int64_t)x * D4) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        const int xj = x0 + j_sub + j_k * stride;
        const float2 mlj = j_k < kReduceBatch && xj < nsplit ? __ldg(ml + xj)
                                                             : make_float2(-INFINITY, 0.f);
        float bm = mlj.x;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, off));
        const float mn = fmaxf(M, bm);
        const float a = M == -INFINITY ? 0.f : exp2f(M - mn);
        const float wj = mlj.x == -INFINITY ? 0.f : exp2f(mlj.x - mn);
        float dj = wj * mlj.y;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) dj += __shfl_xor_sync(0xffffffffu, dj, off);
        den = fmaf(den, a, dj);
        acc.x *= a;
        acc.y *= a;
        acc.z *= a;
        acc.w *= a;
#pragma unroll
        for (int k = 0; k < kReduceBatch; ++k) {
            const float w = __shfl_sync(0xffffffffu, wj, k * rpl + sub);
            acc.x = fmaf(w, v_o[k].x, acc.x);
            acc.y = fmaf(w, v_o[k].y, acc.y);
            acc.z = fmaf(w, v_o[k].z, acc.z);
            acc.w = fmaf(w, v_o[k].w, acc.w);
        }
        M = mn;
    }
    if (rpl == 2) {  // the two half-warps held different rows of the same d
        acc.x += __shfl_xor_sync(0xffffffffu, acc.x, 16);
        acc.y += __shfl_xor_sync(0xffffffffu, acc.y, 16);
        acc.z += __shfl_xor_sync(0xffffffffu, acc.z, 16);
        acc.w += __shfl_xor_sync(0xffffffffu, acc.w, 16);
    }
    float4 *dst = reinterpret_cast<float4 *>(p.out + unit * p.head_dim) + c4;
    if (wpu == 1) {
        if (lane < D4) {
            const float inv = den > 0.f ? 1.f / den : 0.f;
            *dst = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
        }
        return;
    }
    if (lane < D4) acc_s[warp][c4] = acc;
    if (lane == 0) md_s[warp] = make_float2(M, den);
    __threadfence_block();
    __syncwarp();
    const int w0 = warp - wsub;  // the unit's first warp
    int last = 0;
    if (lane == 0) last = atomicAdd(&arrived[w0], 1) == wpu - 1;
    last = __shfl_sync(0xffffffffu, last, 0);
    if (!last) return;
    __threadfence_block();
    if (lane < D4) {
        float mt = -INFINITY;
        for (int w = 0; w < wpu; ++w) mt = fmaxf(mt, md_s[w0 + w].x);
        float4 t = make_float4(0.f, 0.f, 0.f, 0.f);
        float d = 0.f;
        for (int w = 0; w < wpu; ++w) {
            const float2 md = md_s[w0 + w];
            const float sc = md.x == -INFINITY ? 0.f : exp2f(md.x - mt);
            const float4 v = acc_s[w0 + w][c4];
            d = fmaf(sc, md.y, d);
            t.x = fmaf(sc, v.x, t.x);
            t.y = fmaf(sc, v.y, t.y);
            t.z = fmaf(sc, v.z, t.z);
            t.w = fmaf(sc, v.w, t.w);
        }
        const float inv = d > 0.f ? 1.f / d : 0.f;
        *dst = make_float4(t.x * inv, t.y * inv, t.z * inv, t.w * inv);
    }
}

// The same merge for many splits (more than a warp's batch of rows times 4
// warps): one CTA per unit, whose threads own (a group of splits, 4
// consecutive d); the first batch of each thread's partial rows is loaded
// before the weights are formed from the (m, l) pairs, so both loads are in
// flight together.
__global__ void __launch_bounds__(kReduceThreads) decode_reduce_wide_kernel(DecodeParams p) {
    pdl_wait_prior_grid();
    const int h = blockIdx.x, s = blockIdx.y;
    const int L = checked_seq_len(p, s, false);
    const int nsplit = num_splits_for(L, p.partition_size);
    if (nsplit <= 1) return;
    __shared__ float w_s[kMaxSplits];
    __shared__ float red[kReduceThreads / 32];
    __shared__ float4 part[kReduceThreads];
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int64_t u0 = ((int64_t)s * p.num_heads + h) * p.max_splits;
    const float2 *ml = reinterpret_cast<const float2 *>(p.part_ml + 2 * u0);
    const int D4 = p.head_dim / 4;
    const int groups = kReduceThreads / D4;
    const int grp = tid / D4, c4 = tid - grp * D4;
    const float4 *po = reinterpret_cast<const float4 *>(p.part_o + u0 * p.head_dim) + c4;
    float4 v[kReduceBatch];
#pragma unroll
    for (int k = 0; k < kReduceBatch; ++k) {
        const int x = grp + k * groups;
        v[k] = x < nsplit ? __ldg(po + (int64_t)x * D4) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    // max of the split maxima
    float M = -INFINITY;
    for (int x = tid; x < nsplit; x += kReduceThreads) {
        const float2 t = __ldg(ml + x);
        w_s[x] = t.x;
        M = fmaxf(M, t.x);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    if (lane == 0) red[wid] = M;
    __syncthreads();
    M = red[0];
#pragma unroll
    for (int w = 1; w < kReduceThreads / 32; ++w) M = fmaxf(M, red[w]);
    __syncthreads();
    // weights and the denominator
    float den = 0.f;
    for (int x = tid; x < nsplit; x += kReduceThreads) {
        const float wgt = w_s[x] == -INFINITY ? 0.f : exp2f(w_s[x] - M);
        w_s[x] = wgt;
        den = fmaf(wgt, __ldg(ml + x).y, den);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) den += __shfl_xor_sync(0xffffffffu, den, off);
    if (lane == 0) red[wid] = den;
    __syncthreads();
    // numerator: the rows in flight, then any further ones
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int k = 0; k < kReduceBatch; ++k) {
        const int x = grp + k * groups;
        const float wgt = x < nsplit ? w_s[x] : 0.f;
        acc.x = fmaf(wgt, v[k].x, acc.x);
        acc.y = fmaf(wgt, v[k].y, acc.y);
        acc.z = fmaf(wgt, v[k].z, acc.z);
        acc.w = fmaf(wgt, v[k].w, acc.w);
    }
    for (int x = grp + kReduceBatch * groups; x < nsplit; x += groups) {
        const float4 t = __ldg(po + (int64_t)x * D4);
        const float wgt = w_s[x];
        acc.x = fmaf(wgt, t.x, acc.x);
        acc.y = fmaf(wgt, t.y, acc.y);
        acc.z = fmaf(wgt, t.z, acc.z);
        acc.w = fmaf(wgt, t.w, acc.w);
    }
    part[tid] = acc;
    __syncthreads();
    if (tid < D4) {
        float4 tot = part[tid];
        for (int gq = 1; gq < groups; ++gq) {
            const float4 t = part[gq * D4 + tid];
            tot.x += t.x;
            tot.y += t.y;
            tot.z += t.z;
            tot.w += t.w;
        }
        float dsum = 0.f;
#pragma unroll
        for (int w = 0; w < kReduceThreads / 32; ++w) dsum += red[w];
        const float inv = dsum > 0.f ? 1.f / dsum : 0.f;
        float4 *dst = reinterpret_cast<float4 *>(p.out + ((int64_t)s * p.num_heads + h) * p.head_dim);
        dst[tid] = make_float4(tot.x * inv, tot.y * inv, tot.z * inv, tot.w * inv);
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
    // warps per (sequence, query head): enough that a lane holds at most one
    // batch of rows of the longest sequence's splits; beyond 4, the wide form
    const int rpl = 128 / p.head_dim;
    int wpu = 1;
    while (wpu < 8 && wpu * rpl * kReduceBatch < p.max_splits) wpu *= 2;
    const bool wide = wpu == 8;
    const int64_t units = (int64_t)p.num_seqs * p.num_heads;
    const int64_t per_cta = kReduceThreads / 32 / wpu;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = wide ? dim3(p.num_heads, p.num_seqs)
                       : dim3((unsigned)((units + per_cta - 1) / per_cta));
    cfg.blockDim = dim3(kReduceThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (wide) return cudaLaunchKernelEx(&cfg, decode_reduce_wide_kernel, p);
    return cudaLaunchKernelEx(&cfg, decode_reduce_kernel, p, wpu);
}

}  // namespace pa
