// Tensor-core paged decode with one KV head per consumer warp, sm_100a.
//
// The attention is that of mbrenndoerfer.com "Paged Attention > Summary",
// bullet 3 (K/V read through the block table one block at a time, online
// softmax), as in decode_tc.cu; what differs is how a CTA's work is cut.
//
// Work unit: one CTA per (split of `partition_size` tokens, group of W
// adjacent KV heads, sequence).  Consumer warp w owns KV head h0 + w for every
// token of the split, so a warp's running (max, sum, output) is final at the
// end of the split: there is no merge across warps, and a CTA carries W
// heads' work for one start-up (barrier set-up, table slice, first TMA round
// trip).  In the [NB][Hkv][bs][D] cache the W heads of one physical block are
// W*bs contiguous rows, so a single TMA box per 128-byte piece brings a block
// for all of them (blocks of 4 rows are copied by cp.async from all producer
// lanes instead: a 4-row box would start halfway into the 1 KB swizzle atom).
//
// Stage: Ts = max(16, bs) tokens of all W heads; a stage's shared memory
// holds, per 128-byte piece of D, the boxes of its blocks one after another
// (block j of the stage at rows j*W*bs, head w at + w*bs), with the 128B
// swizzle keyed by the token's position mod 8.  Per 16-token tile, a warp
// runs the same products as decode_tc.cu: S^T = K Q^T and O^T += V^T P^T on
// mma.sync m16n8k16 with fp32 accumulation, P in registers as a 16-bit high
// part plus a 16-bit remainder, the softmax online in fp32 in the log2
// domain, tokens past the end masked (logits to -inf, V rows to zero).
//
// Waits are bounded as in decode_tc.cu (~2 s, PA_DEVERR_TIMEOUT, abort flag).
#include <math.h>

#include <cstring>
#include <mutex>

#include "decode_common.cuh"

namespace pa {

namespace hw {

constexpr int kRowBytes = 128;
constexpr int kMaxPartition = 1024;

template <typename T, int D, int BS, int W, int NS>
struct Cfg {
    static constexpr int kThreads = (W + 1) * 32;
    static constexpr bool kAsync = BS < 8;                  // cp.async producer
    static constexpr int kStageTokens = BS < 16 ? 16 : BS;  // per head
    static constexpr int kTiles = kStageTokens / 16;
    static constexpr int kBlocksPerStage = kStageTokens / BS;
    static constexpr int kBoxRows = W * BS;                 // one block, W heads
    static constexpr int kPieces = D / 64;
    static constexpr int kPieceBytes = W * kStageTokens * kRowBytes;
    static constexpr int kKBytes = kPieces * kPieceBytes;
    static constexpr int kStageBytes = 2 * kKBytes;
    static constexpr int kMaxTable = kMaxPartition / BS;
    static constexpr int kBarOffset = NS * kStageBytes;
    static constexpr int kTableOffset = kBarOffset + 2 * NS * 8;
    static constexpr int kFlagOffset = kTableOffset + kMaxTable * 4;
    static constexpr int kSmemBytes = kFlagOffset + 16;
    static constexpr int kDynSmem = kSmemBytes + 1024;  // room to align to 1 KB
    static_assert(kPieceBytes % 1024 == 0, "pieces start on 1 KB swizzle atoms");
    static_assert(kBoxRows <= 256, "a TMA box has at most 256 rows");
    static_assert(sizeof(T) == 2, "16-bit caches");
};

// Row of shared memory holding token `tok` (0 .. Ts-1) of the stage for the
// CTA's head w.
template <int BS, int W>
__device__ __forceinline__ int stage_row(int tok, int w) {
    return (tok / BS) * (W * BS) + w * BS + tok % BS;
}

// Whole-warp bounded wait (lane 0 decides), as in decode_tc.cu.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                          int lane) {
    uint64_t t0 = 0;
    for (uint32_t it = 0;; ++it) {
        const bool ok = mbar_try_wait(bar, parity);
        if (__all_sync(0xffffffffu, ok)) return true;
        if ((it & 63u) == 63u) {
            int quit = 0;
            if (lane == 0) {
                const uint64_t now = global_timer_ns();
                if (t0 == 0) t0 = now;
                quit = (*abort_flag != 0) || (now - t0 > 2000000000ull);
            }
            if (__shfl_sync(0xffffffffu, quit, 0)) return false;
        }
    }
}

template <typename T, int D, int BS, int W, int NS>
__global__ void __launch_bounds__(Cfg<T, D, BS, W, NS>::kThreads)
    decode_hw_kernel(const __grid_constant__ CUtensorMap tmap_k,
                     const __grid_constant__ CUtensorMap tmap_v, const DecodeParams p) {
    using C = Cfg<T, D, BS, W, NS>;
    constexpr int Ts = C::kStageTokens;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

    // launched as a programmatic dependent of the KV append
    pdl_wait_prior_grid();

    const int split = blockIdx.x;
    const int s = seq_of(p, blockIdx.z, split == 0 && blockIdx.y == 0 && threadIdx.x == 0);
    if (s < 0) return;  // uniform over the CTA, before any barrier
    const int h0 = blockIdx.y * W;  // first KV head of the CTA
    const int L = checked_seq_len(p, s, split == 0 && blockIdx.y == 0 && threadIdx.x == 0);
    const int nsplit = num_splits_for(L, p.partition_size);
    if (split >= nsplit) return;  // uniform over the CTA, before any barrier

    const int G = p.num_heads / p.num_kv_heads;
    const int t0 = split * p.partition_size;
    const int t1 = min(L, t0 + p.partition_size);
    const int ntok = max(0, t1 - t0);
    const int nstages = (ntok + Ts - 1) / Ts;
    const int blk0 = t0 / BS;
    const int nblk = (ntok + BS - 1) / BS;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::kBarOffset);
    const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + NS);
    int32_t *table = reinterpret_cast<int32_t *>(smem + C::kTableOffset);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::kFlagOffset);

    if (threadIdx.x == 0) {
        for (int i = 0; i < NS; ++i) {
            mbar_init(full0 + 8 * i, C::kAsync ? 32 : 1);
            mbar_init(empty0 + 8 * i, W);
        }
        *abort_flag = 0;
        fence_mbarrier_init();
    }
    if (warp == W) {
        for (int i = lane; i < nblk; i += 32) {
            const int b = checked_block(p, s, blk0 + i);
            // an entry out of range reads as zeros (rows past the tensor)
            table[i] = b < 0 ? p.num_blocks : b;
        }
    }
    __syncthreads();

    // ------------------------------------------------------------ producer
    if (warp == W) {
        // the fused append: this split holds the new token of the CTA's heads
        if (p.k_new != nullptr && L > 0 && split == nsplit - 1)
            fused_append_rows(p, s, h0, W, L, 2, lane);
        const uint64_t policy = l2_policy_evict_first();
        const uint32_t stage0 = smem_u32(smem);
        if constexpr (C::kAsync) {
            // 16-byte chunks of each block's W*bs contiguous rows, from every
            // lane, into the layout a TMA box would give
            constexpr int kRowChunks = D / 8;
            constexpr int kBlockChunks = C::kBoxRows * kRowChunks;  // per cache
            const char *kc = static_cast<const char *>(p.k_cache);
            const char *vc = static_cast<const char *>(p.v_cache);
            for (int i = 0; i < nstages; ++i) {
                const int buf = i % NS;
                if (i >= NS &&
                    !warp_wait(empty0 + 8 * buf, ((i / NS) - 1) & 1, abort_flag, lane)) {
                    if (lane == 0) {
                        raise_device_error(p.err, PA_DEVERR_TIMEOUT);
                        *abort_flag = 1;
                    }
                    break;
                }
                const int jb = i * C::kBlocksPerStage;
                const int jn = min(C::kBlocksPerStage, nblk - jb);
                const uint32_t kdst = stage0 + buf * C::kStageBytes;
                const uint32_t vdst = kdst + C::kKBytes;
                for (int c = lane; c < jn * kBlockChunks; c += 32) {
                    const int j = c / kBlockChunks, rem = c - j * kBlockChunks;
                    const int rr = rem / kRowChunks, ch = rem - rr * kRowChunks;
                    const int tok = j * BS + rr % BS;
                    const int row = j * C::kBoxRows + rr;
                    const uint32_t off = (ch >> 3) * C::kPieceBytes + row * kRowBytes +
                                         (((ch & 7) ^ (tok & 7)) << 4);
                    const int b = table[jb + j];
                    const bool ok = b < p.num_blocks;
                    const int64_t src =
                        ((((int64_t)(ok ? b : 0) * p.num_kv_heads + h0) * BS + rr) * D + ch * 8) *
                        2;
                    cp_async_16(kdst + off, kc + src, ok ? 16u : 0u, policy);
                    cp_async_16(vdst + off, vc + src, ok ? 16u : 0u, policy);
                }
                cp_async_arrive_noinc(full0 + 8 * buf);
            }
            cp_async_wait_all();  // copies in flight land before the CTA exits
        } else if (lane == 0) {
            prefetch_tensormap(&tmap_k);
            prefetch_tensormap(&tmap_v);
            int issued = 0;
            for (int i = 0; i < nstages; ++i) {
                const int buf = i % NS;
                if (i >= NS &&
                    !mbar_wait_bounded(empty0 + 8 * buf, ((i / NS) - 1) & 1, abort_flag)) {
                    raise_device_error(p.err, PA_DEVERR_TIMEOUT);
                    *abort_flag = 1;
                    break;
                }
                const int jb = i * C::kBlocksPerStage;
                const int jn = min(C::kBlocksPerStage, nblk - jb);
                const uint32_t full = full0 + 8 * buf;
                mbar_arrive_expect_tx(full, (uint32_t)(jn * C::kPieces * C::kBoxRows * kRowBytes * 2));
                const uint32_t kdst = stage0 + buf * C::kStageBytes;
                const uint32_t vdst = kdst + C::kKBytes;
                for (int j = 0; j < jn; ++j) {
                    const int y = (table[jb + j] * p.num_kv_heads + h0) * BS;
#pragma unroll
                    for (int pc = 0; pc < C::kPieces; ++pc) {
                        const uint32_t off = pc * C::kPieceBytes + j * C::kBoxRows * kRowBytes;
                        tma_load_2d(kdst + off, &tmap_k, pc * 64, y, full, policy);
                        tma_load_2d(vdst + off, &tmap_v, pc * 64, y, full, policy);
                    }
                }
                issued = i + 1;
            }
            // copies in flight land before the CTA exits
            for (int i = max(0, issued - NS); i < issued; ++i)
                mbar_wait_bounded(full0 + 8 * (i % NS), (i / NS) & 1, nullptr);
        }
        return;
    }

    // ------------------------------------------------------------ consumers
    // warp w: KV head h0 + w, query heads (h0 + w) * G .. + G - 1
    const int gid = lane >> 2, tig = lane & 3;
    const int hq0 = (h0 + warp) * G;
    uint32_t qb[D / 16][2];
    {
        const T *qrow = static_cast<const T *>(p.q) + ((int64_t)s * p.num_heads + hq0 + gid) * D;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            if (gid < G) {
                qb[kk][0] = __ldg(reinterpret_cast<const uint32_t *>(qrow + 16 * kk + 2 * tig));
                qb[kk][1] = __ldg(reinterpret_cast<const uint32_t *>(qrow + 16 * kk + 8 + 2 * tig));
            } else {
                qb[kk][0] = qb[kk][1] = 0u;
            }
        }
    }

    float m_run[2] = {-INFINITY, -INFINITY};
    float l_run[2] = {0.f, 0.f};
    float o[D / 16][4];
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;

    const int r7 = lane & 7;
    const int tk_k = r7 + ((lane >> 3) & 1) * 8;  // token of the tile this lane addresses (K)
    const int chk_k = lane >> 4;
    const int tk_v = r7 + (lane >> 4) * 8;        // (V, transposed)
    const int chk_v = (lane >> 3) & 1;
    const float sl2 = p.scale_log2;
    const uint32_t stage0 = smem_u32(smem);

    for (int i = 0; i < nstages; ++i) {
        const int buf = i % NS;
        if (!warp_wait(full0 + 8 * buf, (i / NS) & 1, abort_flag, lane)) {
            if (lane == 0) {
                raise_device_error(p.err, PA_DEVERR_TIMEOUT);
                *abort_flag = 1;
            }
            break;
        }
        const uint32_t kbase = stage0 + buf * C::kStageBytes;
        const uint32_t vbase = kbase + C::kKBytes;
#pragma unroll
        for (int t = 0; t < C::kTiles; ++t) {
            const int tb = t0 + i * Ts + 16 * t;
            if (tb >= t1) break;
            const uint32_t rk = stage_row<BS, W>(16 * t + tk_k, warp) * kRowBytes;
            const uint32_t rv = stage_row<BS, W>(16 * t + tk_v, warp) * kRowBytes;
            // ---- S^T = K Q^T (two accumulators shorten the MMA chain)
            float c[4] = {0.f, 0.f, 0.f, 0.f}, c2[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const int chunk = ((kk & 3) << 1) + chk_k;
                const uint32_t addr = kbase + (kk >> 2) * C::kPieceBytes + rk + ((chunk ^ r7) << 4);
                uint32_t a[4];
                ldmatrix_x4(addr, a[0], a[1], a[2], a[3]);
                Mma<T>::run((kk & 1) ? c2 : c, a, qb[kk][0], qb[kk][1]);
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) c[e] += c2[e];
            // ---- online softmax (log2 domain); tokens past the end -> -inf
            const bool ok_lo = tb + gid < t1, ok_hi = tb + gid + 8 < t1;
            const float x0 = ok_lo ? c[0] * sl2 : -INFINITY;
            const float x1 = ok_lo ? c[1] * sl2 : -INFINITY;
            const float x2 = ok_hi ? c[2] * sl2 : -INFINITY;
            const float x3 = ok_hi ? c[3] * sl2 : -INFINITY;
            float mx0 = fmaxf(x0, x2), mx1 = fmaxf(x1, x3);
#pragma unroll
            for (int off = 4; off < 32; off <<= 1) {
                mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
                mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
            }
            const float mn0 = fmaxf(m_run[0], mx0), mn1 = fmaxf(m_run[1], mx1);
            const float al0 = exp2f(m_run[0] - mn0), al1 = exp2f(m_run[1] - mn1);
            m_run[0] = mn0;
            m_run[1] = mn1;
            const float p0 = exp2f(x0 - mn0), p1 = exp2f(x1 - mn1);
            const float p2 = exp2f(x2 - mn0), p3 = exp2f(x3 - mn1);
            // P = P_hi + P_lo, both 16-bit
            const uint32_t plo = Mma<T>::pack(p0, p1);
            const uint32_t phi = Mma<T>::pack(p2, p3);
            const uint32_t rlo = Mma<T>::pack(p0 - Mma<T>::lo(plo), p1 - Mma<T>::hi(plo));
            const uint32_t rhi = Mma<T>::pack(p2 - Mma<T>::lo(phi), p3 - Mma<T>::hi(phi));
            l_run[0] = l_run[0] * al0 + (p0 + p2);
            l_run[1] = l_run[1] * al1 + (p1 + p3);
#pragma unroll
            for (int mt = 0; mt < D / 16; ++mt) {
                o[mt][0] *= al0;
                o[mt][1] *= al1;
                o[mt][2] *= al0;
                o[mt][3] *= al1;
            }
            const uint32_t pb0 = movmatrix_trans(plo);
            const uint32_t pb1 = movmatrix_trans(phi);
            const uint32_t pr0 = movmatrix_trans(rlo);
            const uint32_t pr1 = movmatrix_trans(rhi);
            // rows past the end may hold stale data: zero them so 0 * x stays 0
            uint32_t vm0 = 0xffffffffu, vm1 = 0xffffffffu;
            if (tb + 16 > t1) {
                const int te = t1 - tb;
                vm0 = (2 * tig < te ? 0x0000ffffu : 0u) | (2 * tig + 1 < te ? 0xffff0000u : 0u);
                vm1 = (2 * tig + 8 < te ? 0x0000ffffu : 0u) | (2 * tig + 9 < te ? 0xffff0000u : 0u);
            }
            // ---- O^T += V^T P^T
#pragma unroll
            for (int mt = 0; mt < D / 16; ++mt) {
                const int chunk = ((mt & 3) << 1) + chk_v;
                const uint32_t addr = vbase + (mt >> 2) * C::kPieceBytes + rv + ((chunk ^ r7) << 4);
                uint32_t a[4];
                ldmatrix_x4_trans(addr, a[0], a[1], a[2], a[3]);
                a[0] &= vm0;
                a[1] &= vm0;
                a[2] &= vm1;
                a[3] &= vm1;
                Mma<T>::run(o[mt], a, pb0, pb1);
                Mma<T>::run(o[mt], a, pr0, pr1);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty0 + 8 * buf);
    }

    // ------------------------------------------------------------ output
    // the 8 lanes of a head pair (one per gid) hold disjoint tokens' sums
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
        l_run[0] += __shfl_xor_sync(0xffffffffu, l_run[0], off);
        l_run[1] += __shfl_xor_sync(0xffffffffu, l_run[1], off);
    }
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        const int hh = 2 * tig + e;  // query head within the group
        if (hh < G) {
            const int hq = hq0 + hh;
            if (nsplit == 1) {
                const float inv = l_run[e] > 0.f ? 1.f / l_run[e] : 0.f;
                float *dst = p.out + ((int64_t)s * p.num_heads + hq) * D;
#pragma unroll
                for (int mt = 0; mt < D / 16; ++mt) {
                    dst[16 * mt + gid] = o[mt][e] * inv;
                    dst[16 * mt + gid + 8] = o[mt][2 + e] * inv;
                }
            } else {
                const int64_t u = ((int64_t)s * p.num_heads + hq) * p.max_splits + split;
                float *dst = p.part_o + u * D;
#pragma unroll
                for (int mt = 0; mt < D / 16; ++mt) {
                    dst[16 * mt + gid] = o[mt][e];
                    dst[16 * mt + gid + 8] = o[mt][2 + e];
                }
                if (gid == 0) {
                    p.part_ml[2 * u] = m_run[e];
                    p.part_ml[2 * u + 1] = l_run[e];
                }
            }
        }
    }
    if (p.tickets != nullptr && nsplit > 1) {
        // the CTA of this (sequence, head group) to finish last merges the splits
        __threadfence();
        named_barrier_sync(1, W * 32);
        volatile int *last = abort_flag + 1;
        if (threadIdx.x == 0)
            *last = ticket_arrive_last(p.tickets + (int64_t)s * p.num_kv_heads + h0, p.tag, nsplit);
        named_barrier_sync(1, W * 32);
        if (*last) merge_splits(p, s, h0 * G, W * G, nsplit, threadIdx.x, W * 32);
    }
    pdl_launch_dependents();
}

template <typename T, int D, int BS, int W, int NS>
static cudaError_t launch_inst(const DecodeParams &p, const CUtensorMap &mk, const CUtensorMap &mv,
                               cudaStream_t stream) {
    using C = Cfg<T, D, BS, W, NS>;
    static std::once_flag once[64];
    static cudaError_t attr_err[64];
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::call_once(once[dev], [&] {
        attr_err[dev] = cudaFuncSetAttribute(decode_hw_kernel<T, D, BS, W, NS>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             C::kDynSmem);
    });
    if (attr_err[dev] != cudaSuccess) return attr_err[dev];
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.max_splits, p.num_kv_heads / W, p.num_seqs);
    cfg.blockDim = dim3(C::kThreads);
    cfg.dynamicSmemBytes = C::kDynSmem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_hw_kernel<T, D, BS, W, NS>, mk, mv, p);
}

// Ring depth per shape: about 32 KB of stages for one or two heads per CTA,
// 64 KB for four (a stage is Ts tokens x W heads x D x 2 bytes x 2 caches).
template <typename T, int D, int BS, int W>
static cudaError_t launch_w(const DecodeParams &p, const CUtensorMap &mk, const CUtensorMap &mv,
                            cudaStream_t stream) {
    constexpr int kStage = 2 * (D / 64) * W * (BS < 16 ? 16 : BS) * kRowBytes;
    constexpr int NS = kStage >= 32768 ? 2 : (32768 / kStage < 4 ? 32768 / kStage : 4);
    return launch_inst<T, D, BS, W, NS>(p, mk, mv, stream);
}

// A stage holds at most 64 token rows per piece (W heads x Ts tokens), so
// that the ring stays within 64 KB at D = 128: W up to 4 for blocks of up to
// 16 rows, 2 for 32, 1 for 64.
template <typename T, int D, int BS>
static cudaError_t launch_bs(const DecodeParams &p, int W, const CUtensorMap &mk,
                             const CUtensorMap &mv, cudaStream_t stream) {
    constexpr int Ts = BS < 16 ? 16 : BS;
    switch (W) {
    case 1: return launch_w<T, D, BS, 1>(p, mk, mv, stream);
    case 2:
        if constexpr (2 * Ts <= 64) return launch_w<T, D, BS, 2>(p, mk, mv, stream);
        return cudaErrorNotSupported;
    case 4:
        if constexpr (4 * Ts <= 64) return launch_w<T, D, BS, 4>(p, mk, mv, stream);
        return cudaErrorNotSupported;
    default: return cudaErrorNotSupported;
    }
}

template <typename T, int D>
static cudaError_t launch_d(const DecodeParams &p, int W, const CUtensorMap &mk,
                            const CUtensorMap &mv, cudaStream_t stream) {
    switch (p.block_size) {
    case 4: return launch_bs<T, D, 4>(p, W, mk, mv, stream);
    case 8: return launch_bs<T, D, 8>(p, W, mk, mv, stream);
    case 16: return launch_bs<T, D, 16>(p, W, mk, mv, stream);
    case 32: return launch_bs<T, D, 32>(p, W, mk, mv, stream);
    case 64: return launch_bs<T, D, 64>(p, W, mk, mv, stream);
    default: return cudaErrorNotSupported;
    }
}

}  // namespace hw

namespace hw {
// CTAs of an instance resident per SM (its shared-memory attribute set first,
// as launch_inst does), or -1.
template <typename T, int D, int BS, int W>
static int resident_w() {
    constexpr int kStage = 2 * (D / 64) * W * (BS < 16 ? 16 : BS) * kRowBytes;
    constexpr int NS = kStage >= 32768 ? 2 : (32768 / kStage < 4 ? 32768 / kStage : 4);
    using C = Cfg<T, D, BS, W, NS>;
    if (cudaFuncSetAttribute(decode_hw_kernel<T, D, BS, W, NS>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, C::kDynSmem) != cudaSuccess)
        return -1;
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_hw_kernel<T, D, BS, W, NS>,
                                                      C::kThreads, C::kDynSmem) != cudaSuccess)
        return -1;
    return n;
}
template <typename T, int D>
static int resident_d(int block_size) {
    switch (block_size) {
    case 8: return resident_w<T, D, 8, 2>();
    case 16: return resident_w<T, D, 16, 2>();
    default: return -1;
    }
}
}  // namespace hw

int decode_hw2_resident_per_sm(int dtype, int head_dim, int block_size) {
    if (dtype != PA_BF16 && dtype != PA_F16) return -1;
    if (head_dim != 64 && head_dim != 128) return -1;
    if (dtype == PA_BF16)
        return head_dim == 128 ? hw::resident_d<__nv_bfloat16, 128>(block_size)
                               : hw::resident_d<__nv_bfloat16, 64>(block_size);
    return head_dim == 128 ? hw::resident_d<__half, 128>(block_size)
                           : hw::resident_d<__half, 64>(block_size);
}

cudaError_t launch_decode_hw(const DecodeParams &p, int dtype, int heads_per_cta,
                             cudaStream_t stream) {
    if (dtype != PA_BF16 && dtype != PA_F16) return cudaErrorNotSupported;
    if (p.head_dim != 64 && p.head_dim != 128) return cudaErrorNotSupported;
    if (p.partition_size % 64 != 0 || p.partition_size > hw::kMaxPartition)
        return cudaErrorNotSupported;
    if (p.num_heads / p.num_kv_heads > 8) return cudaErrorNotSupported;
    const int W = heads_per_cta;
    const int Ts = p.block_size < 16 ? 16 : p.block_size;
    if ((W != 1 && W != 2 && W != 4) || p.num_kv_heads % W != 0 || W * Ts > 64)
        return cudaErrorNotSupported;
    if (p.num_seqs == 0) return cudaSuccess;
    CUtensorMap mk, mv;
    std::memset(&mk, 0, sizeof(mk));
    std::memset(&mv, 0, sizeof(mv));
    if (p.block_size >= 8) {
        const int64_t rows = (int64_t)p.num_blocks * p.num_kv_heads * p.block_size;
        if (!make_cache_tensor_map(&mk, p.k_cache, dtype, p.head_dim, rows, W * p.block_size) ||
            !make_cache_tensor_map(&mv, p.v_cache, dtype, p.head_dim, rows, W * p.block_size))
            return cudaErrorInvalidValue;
    }
    if (dtype == PA_BF16)
        return p.head_dim == 128 ? hw::launch_d<__nv_bfloat16, 128>(p, W, mk, mv, stream)
                                 : hw::launch_d<__nv_bfloat16, 64>(p, W, mk, mv, stream);
    return p.head_dim == 128 ? hw::launch_d<__half, 128>(p, W, mk, mv, stream)
                             : hw::launch_d<__half, 64>(p, W, mk, mv, stream);
}

}  // namespace pa
