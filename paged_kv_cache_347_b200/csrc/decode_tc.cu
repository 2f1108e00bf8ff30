// Tensor-core paged decode for 16-bit caches (bf16 / f16), sm_100a.
//
// What it computes is the attention of mbrenndoerfer.com "Paged Attention >
// Summary", bullet 3: keys and values read through the block table one block
// at a time, no gather into a contiguous buffer, softmax kept online.  It is a
// memory-bound kernel -- every K/V byte is read once -- so the design is
// about keeping HBM busy.
//
// Work unit: one CTA per (split of `partition_size` tokens, KV head g,
// sequence s); W consumer warps + 1 producer warp, several CTAs per SM.
// Several small CTAs per SM beat one persistent CTA per SM here: each CTA has
// its own producer issuing TMA loads, and with 6 CTAs per SM their loads
// overlap each other's start-up and merge phases.
//
//  * Producer (one thread): copies the CTA's slice of the block table into
//    shared memory, then streams the split in stages of 16*W tokens through a
//    ring of NS stage buffers.  For each physical block of a stage it issues
//    TMA tensor loads (no multicast) of the block's K and V rows for head g --
//    a (block, head) run is bs*D contiguous elements of the [NB][Hkv][bs][D]
//    cache -- as 128-byte-wide boxes with the 128B swizzle, completion
//    counted in bytes on the stage's "full" mbarrier, with an L2 evict-first
//    hint (K/V are read once).  A buffer is refilled after the consumer warps
//    release it on its "empty" mbarrier.
//
//  * Consumers: warp w owns tokens [16w, 16w+16) of every stage.  The GQA
//    group is a genuine dense tile, so both products run on mma.sync
//    m16n8k16 with fp32 accumulation:
//      S^T[16 tok x 8 heads] = K[16 x D] . Q^T[D x 8]      (A = K via ldmatrix)
//      O^T[D x 8 heads]     += V^T[D x 16] . P^T[16 x 8]    (A = V via ldmatrix.trans)
//    The QK accumulator fragment holds, per lane, 2 tokens x 2 heads; it is
//    rounded to 16 bits and transposed in registers with movmatrix into the
//    B fragment of the PV product, so P never touches shared memory.  P is
//    split into a 16-bit high part and a 16-bit remainder and the PV product
//    is issued for both, so the weights carry ~16 significant bits (one bf16
//    rounding of P alone costs up to 2^-9 relative, which the 3e-3 output
//    bound cannot absorb on short contexts).  Heads beyond G are zero rows of
//    Q.  Each lane's O fragment covers the same 2 heads as its S fragment, so
//    the online-softmax rescale is per lane.  Running max (log2 units) and
//    running sum stay in fp32.
//
//  * End: the warps' (m, l, O) are merged through shared memory (the drained
//    stage buffers) and the CTA writes either the normalised output (one
//    split) or the partial for the reduce kernel.
//
// All pipeline waits are bounded (~2 s); a wait that gives up sets
// PA_DEVERR_TIMEOUT and an abort flag the other warps observe, and the
// producer waits (bounded) for its own copies in flight before it exits.
#include <math.h>

#include <mutex>

#include "decode_common.cuh"

namespace pa {

namespace tc {

constexpr int kRowBytes = 128;  // one swizzled box row
constexpr int kMaxPartition = 1024;
constexpr int kMaxG = 8;

template <typename T, int D, int BS, int W, int NS>
struct Cfg {
    static constexpr int kThreads = (W + 1) * 32;
    // blocks of 4 rows are staged by cp.async from all producer lanes: a TMA
    // box of 4 rows would start halfway into the 1 KB 128B-swizzle atom
    static constexpr bool kAsync = BS < 8;
    static constexpr int kStageTokens = 16 * W;
    static constexpr int kPieces = D / 64;                        // 128-byte pieces of a row
    static constexpr int kPieceBytes = kStageTokens * kRowBytes;
    static constexpr int kKBytes = kPieces * kPieceBytes;         // K of one stage
    static constexpr int kStageBytes = 2 * kKBytes;               // K + V
    static constexpr int kBlocksPerStage = kStageTokens / BS;
    static constexpr int kMaxTable = kMaxPartition / BS;
    static constexpr int kMergeStride = D + 4;                    // floats per head row
    static constexpr int kMergeBytes = W * kMaxG * kMergeStride * 4;
    static constexpr int kBarOffset = NS * kStageBytes;
    static constexpr int kTableOffset = kBarOffset + 2 * NS * 8;
    static constexpr int kAbortOffset = kTableOffset + kMaxTable * 4;
    static constexpr int kMlOffset = kAbortOffset + 16;           // m, l of the merge
    static constexpr int kSmemBytes = kMlOffset + 2 * W * kMaxG * 4;
    static constexpr int kDynSmem = kSmemBytes + 1024;            // room to align to 1 KB
    static_assert(kMergeBytes <= NS * kStageBytes, "merge area reuses the stage buffers");
    static_assert(kStageTokens % BS == 0, "block size divides a stage");
    static_assert(kPieceBytes % 1024 == 0, "TMA boxes need 1 KB-aligned destinations");
    static_assert(sizeof(T) == 2, "16-bit caches");
};

// Waits, as a whole warp, for the phase of `bar` with parity `parity`; the
// decision to give up is lane 0's, so the outcome is warp-uniform.
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
    decode_tc_kernel(const __grid_constant__ CUtensorMap tmap_k,
                     const __grid_constant__ CUtensorMap tmap_v, const DecodeParams p) {
    using C = Cfg<T, D, BS, W, NS>;
    constexpr int kStageTokens = C::kStageTokens;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

    // launched as a programmatic dependent: the previous kernel on the stream
    // (e.g. the KV append) must be complete before any input is read
    pdl_wait_prior_grid();

    const int split = blockIdx.x, g = blockIdx.y;
    const int s = seq_of(p, blockIdx.z, split == 0 && g == 0 && threadIdx.x == 0);
    if (s < 0) return;  // uniform over the CTA, before any barrier
    const int L = checked_seq_len(p, s, split == 0 && g == 0 && threadIdx.x == 0);
    const int nsplit = num_splits_for(L, p.partition_size);
    if (split >= nsplit) return;  // uniform over the CTA, before any barrier

    const int G = p.num_heads / p.num_kv_heads;
    const int t0 = split * p.partition_size;
    const int t1 = min(L, t0 + p.partition_size);
    const int ntok = max(0, t1 - t0);
    const int nstages = (ntok + kStageTokens - 1) / kStageTokens;
    const int blk0 = t0 / BS;
    const int nblk = (ntok + BS - 1) / BS;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::kBarOffset);
    const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + NS);
    int32_t *table = reinterpret_cast<int32_t *>(smem + C::kTableOffset);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::kAbortOffset);

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
            // an entry out of range reads rows past the tensor: TMA fills zeros
            table[i] = b < 0 ? p.num_blocks : b;
        }
    }
    __syncthreads();

    // ------------------------------------------------------------ producer
    // the fused append: this split holds the new token, whose row the loads
    // below then read
    if (warp == W && p.k_new != nullptr && L > 0 && split == nsplit - 1)
        fused_append_rows(p, s, g, 1, L, 2, lane);
    if (C::kAsync && warp == W) {
        // every lane copies 16-byte chunks of the stage's (block, head) rows
        // into the layout the TMA boxes give (row r of a 1 KB-aligned piece,
        // chunk c at c ^ (r mod 8)), then arrives on the stage's barrier once
        // its copies have landed
        constexpr int kRowChunks = D / 8;              // 16-byte chunks per row
        constexpr int kBlockChunks = BS * kRowChunks;  // per cache
        const uint64_t policy = l2_policy_evict_first();
        const uint32_t stage0 = smem_u32(smem);
        const char *kc = static_cast<const char *>(p.k_cache);
        const char *vc = static_cast<const char *>(p.v_cache);
        for (int i = 0; i < nstages; ++i) {
            const int buf = i % NS;
            if (i >= NS && !warp_wait(empty0 + 8 * buf, ((i / NS) - 1) & 1, abort_flag, lane)) {
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
                const int r = rem / kRowChunks, ch = rem - r * kRowChunks;
                const int row = j * BS + r;
                const uint32_t off = (ch >> 3) * C::kPieceBytes + row * kRowBytes +
                                     (((ch & 7) ^ (row & 7)) << 4);
                // an entry out of range (marked num_blocks) reads as zeros
                const int b = table[jb + j];
                const bool ok = b < p.num_blocks;
                const int64_t src = ((((int64_t)(ok ? b : 0) * p.num_kv_heads + g) * BS + r) * D +
                                     ch * 8) * 2;
                cp_async_16(kdst + off, kc + src, ok ? 16u : 0u, policy);
                cp_async_16(vdst + off, vc + src, ok ? 16u : 0u, policy);
            }
            cp_async_arrive_noinc(full0 + 8 * buf);
        }
        // copies still in flight must land before the CTA may exit
        cp_async_wait_all();
        return;
    }
    if (warp == W) {
        if (lane == 0) {
            prefetch_tensormap(&tmap_k);
            prefetch_tensormap(&tmap_v);
            const uint64_t policy = l2_policy_evict_first();
            const uint32_t stage0 = smem_u32(smem);
            int issued = 0;
            for (int i = 0; i < nstages; ++i) {
                const int buf = i % NS;
                if (i >= NS && !mbar_wait_bounded(empty0 + 8 * buf, ((i / NS) - 1) & 1, abort_flag)) {
                    raise_device_error(p.err, PA_DEVERR_TIMEOUT);
                    *abort_flag = 1;
                    break;
                }
                const int jb = i * C::kBlocksPerStage;
                const int jn = min(C::kBlocksPerStage, nblk - jb);
                const uint32_t full = full0 + 8 * buf;
                mbar_arrive_expect_tx(full, (uint32_t)(jn * 4 * BS * D));
                const uint32_t kdst = stage0 + buf * C::kStageBytes;
                const uint32_t vdst = kdst + C::kKBytes;
                for (int j = 0; j < jn; ++j) {
                    const int y = (table[jb + j] * p.num_kv_heads + g) * BS;
#pragma unroll
                    for (int pc = 0; pc < C::kPieces; ++pc) {
                        const uint32_t off = pc * C::kPieceBytes + j * BS * kRowBytes;
                        tma_load_2d(kdst + off, &tmap_k, pc * 64, y, full, policy);
                        tma_load_2d(vdst + off, &tmap_v, pc * 64, y, full, policy);
                    }
                }
                issued = i + 1;
            }
            // copies still in flight must land before the CTA may exit
            for (int i = max(0, issued - NS); i < issued; ++i)
                mbar_wait_bounded(full0 + 8 * (i % NS), (i / NS) & 1, nullptr);
        }
        return;
    }

    // ------------------------------------------------------------ consumers
    const int gid = lane >> 2, tig = lane & 3;
    uint32_t qb[D / 16][2];
    {
        const T *qrow = static_cast<const T *>(p.q) + ((int64_t)s * p.num_heads + g * G + gid) * D;
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

    // ldmatrix row addresses: rows are tokens of this warp's 16-token tile
    const int r7 = lane & 7;
    const int row_k = 16 * warp + r7 + ((lane >> 3) & 1) * 8;
    const int chk_k = lane >> 4;
    const int row_v = 16 * warp + r7 + (lane >> 4) * 8;
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
        const int tb = t0 + i * kStageTokens + 16 * warp;
        if (tb < t1) {
            const uint32_t kbase = stage0 + buf * C::kStageBytes;
            const uint32_t vbase = kbase + C::kKBytes;
            // ---- S^T = K Q^T (two accumulators shorten the MMA chain)
            float c[4] = {0.f, 0.f, 0.f, 0.f}, c2[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const int chunk = ((kk & 3) << 1) + chk_k;
                const uint32_t addr = kbase + (kk >> 2) * C::kPieceBytes + row_k * kRowBytes +
                                      ((chunk ^ r7) << 4);
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
            const uint32_t plo = Mma<T>::pack(p0, p1);  // tokens 0-7 (high part)
            const uint32_t phi = Mma<T>::pack(p2, p3);  // tokens 8-15
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
                const uint32_t addr = vbase + (mt >> 2) * C::kPieceBytes + row_v * kRowBytes +
                                      ((chunk ^ r7) << 4);
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

    // ------------------------------------------------------------ merge
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
        l_run[0] += __shfl_xor_sync(0xffffffffu, l_run[0], off);
        l_run[1] += __shfl_xor_sync(0xffffffffu, l_run[1], off);
    }
    named_barrier_sync(1, W * 32);  // every stage buffer has been read
    float *mo = reinterpret_cast<float *>(smem);  // [warp][8 heads][D + 4]
    float *mml = reinterpret_cast<float *>(smem + C::kMlOffset);  // m[warp][8], l[warp][8]
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt) {
        float *w0 = mo + (warp * kMaxG + 2 * tig) * C::kMergeStride + 16 * mt + gid;
        float *w1 = w0 + C::kMergeStride;
        w0[0] = o[mt][0];
        w1[0] = o[mt][1];
        w0[8] = o[mt][2];
        w1[8] = o[mt][3];
    }
    if (gid == 0) {
        mml[warp * kMaxG + 2 * tig] = m_run[0];
        mml[warp * kMaxG + 2 * tig + 1] = m_run[1];
        mml[W * kMaxG + warp * kMaxG + 2 * tig] = l_run[0];
        mml[W * kMaxG + warp * kMaxG + 2 * tig + 1] = l_run[1];
    }
    named_barrier_sync(1, W * 32);
    for (int idx = threadIdx.x; idx < G * D; idx += W * 32) {
        const int h = idx / D, d = idx - (idx / D) * D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < W; ++w) M = fmaxf(M, mml[w * kMaxG + h]);
        float num = 0.f, den = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < W; ++w) {
                const float sc = exp2f(mml[w * kMaxG + h] - M);
                num = fmaf(sc, mo[(w * kMaxG + h) * C::kMergeStride + d], num);
                den = fmaf(sc, mml[W * kMaxG + w * kMaxG + h], den);
            }
        }
        store_unit(p, s, g * G + h, split, nsplit, d, M, den, num);
    }
    if (p.tickets != nullptr && nsplit > 1) {
        // the CTA of this (sequence, KV head) to finish last merges the splits
        __threadfence();
        named_barrier_sync(1, W * 32);
        volatile int *last = abort_flag + 1;
        if (threadIdx.x == 0)
            *last = ticket_arrive_last(p.tickets + (int64_t)s * p.num_kv_heads + g, p.tag, nsplit);
        named_barrier_sync(1, W * 32);
        if (*last) merge_splits(p, s, g * G, G, nsplit, threadIdx.x, W * 32);
    }
    // this CTA's outputs are written: a dependent kernel may begin launching
    pdl_launch_dependents();
}

// ------------------------------------------------------------ host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = []() -> EncodeTiledFn {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        return reinterpret_cast<EncodeTiledFn>(ptr);
    }();
    return fn;
}

}  // namespace tc

// Rows of 128 bytes (64 elements), `box_rows` rows per box, over the cache
// viewed as a [NB*Hkv*bs][D] matrix, 128B swizzle.
bool make_cache_tensor_map(CUtensorMap *m, const void *base, int dtype, int D, int64_t rows,
                           int box_rows) {
    using tc::EncodeTiledFn;
    using tc::encode_fn;
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)D * 2};
    const cuuint32_t box[2] = {64u, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1u, 1u};
    const CUtensorMapDataType dt =
        dtype == PA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    return enc(m, dt, 2, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace tc {

template <typename T, int D, int BS, int W, int NS>
static cudaError_t launch_tc_inst(const DecodeParams &p, const CUtensorMap &mk,
                                  const CUtensorMap &mv, cudaStream_t stream) {
    using C = Cfg<T, D, BS, W, NS>;
    static std::once_flag once[64];
    static cudaError_t attr_err[64];
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::call_once(once[dev], [&] {
        attr_err[dev] = cudaFuncSetAttribute(decode_tc_kernel<T, D, BS, W, NS>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             C::kDynSmem);
    });
    if (attr_err[dev] != cudaSuccess) return attr_err[dev];
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.max_splits, p.num_kv_heads, p.num_seqs);
    cfg.blockDim = dim3(C::kThreads);
    cfg.dynamicSmemBytes = C::kDynSmem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_tc_kernel<T, D, BS, W, NS>, mk, mv, p);
}

// 2 consumer warps (32-token stages); 2 stages of 16 KB for D = 128 and 4 of
// 8 KB for D = 64: ~34 KB of shared memory, 6 CTAs (18 warps) per SM.  On the
// 32k-token batch this beat 4 warps x 2-3 stages (3 or 2 CTAs per SM) and one
// persistent CTA per SM: more independent producers keep more TMA loads in
// flight.
template <typename T, int D>
static cudaError_t launch_tc_d(const DecodeParams &p, const CUtensorMap &mk,
                               const CUtensorMap &mv, cudaStream_t stream) {
    constexpr int W = 2;
    constexpr int NS = D == 128 ? 2 : 4;
    switch (p.block_size) {
    case 4: return launch_tc_inst<T, D, 4, W, NS>(p, mk, mv, stream);
    case 8: return launch_tc_inst<T, D, 8, W, NS>(p, mk, mv, stream);
    case 16: return launch_tc_inst<T, D, 16, W, NS>(p, mk, mv, stream);
    case 32: return launch_tc_inst<T, D, 32, W, NS>(p, mk, mv, stream);
    // a 64-token block fills a 4-warp stage (64 KB at D = 128: 3 CTAs per SM)
    case 64: return launch_tc_inst<T, D, 64, 4, D == 128 ? 2 : 4>(p, mk, mv, stream);
    default: return cudaErrorNotSupported;
    }
}

// CTAs of one instance resident per SM (the launch's shared-memory attribute
// set first, as launch_tc_inst does), or -1.
template <typename T, int D, int BS, int W, int NS>
static int resident_inst() {
    using C = Cfg<T, D, BS, W, NS>;
    if (cudaFuncSetAttribute(decode_tc_kernel<T, D, BS, W, NS>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C::kDynSmem) != cudaSuccess)
        return -1;
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_tc_kernel<T, D, BS, W, NS>,
                                                      C::kThreads, C::kDynSmem) != cudaSuccess)
        return -1;
    return n;
}

// the instances launch_tc_d picks
template <typename T, int D>
static int resident_d(int block_size) {
    constexpr int NS = D == 128 ? 2 : 4;
    switch (block_size) {
    case 4: return resident_inst<T, D, 4, 2, NS>();
    case 8: return resident_inst<T, D, 8, 2, NS>();
    case 16: return resident_inst<T, D, 16, 2, NS>();
    case 32: return resident_inst<T, D, 32, 2, NS>();
    case 64: return resident_inst<T, D, 64, 4, D == 128 ? 2 : 4>();
    default: return -1;
    }
}

}  // namespace tc

int decode_tc_resident_per_sm(int dtype, int head_dim, int block_size) {
    if (dtype != PA_BF16 && dtype != PA_F16) return -1;
    if (head_dim != 64 && head_dim != 128) return -1;
    if (dtype == PA_BF16)
        return head_dim == 128 ? tc::resident_d<__nv_bfloat16, 128>(block_size)
                               : tc::resident_d<__nv_bfloat16, 64>(block_size);
    return head_dim == 128 ? tc::resident_d<__half, 128>(block_size)
                           : tc::resident_d<__half, 64>(block_size);
}

cudaError_t launch_decode_tc(const DecodeParams &p, int dtype, cudaStream_t stream) {
    if (dtype != PA_BF16 && dtype != PA_F16) return cudaErrorNotSupported;
    if (p.block_size < 4 || p.block_size > 64) return cudaErrorNotSupported;
    if (p.head_dim != 64 && p.head_dim != 128) return cudaErrorNotSupported;
    if (p.partition_size % 64 != 0 || p.partition_size > tc::kMaxPartition)
        return cudaErrorNotSupported;
    if (p.num_heads / p.num_kv_heads > tc::kMaxG) return cudaErrorNotSupported;
    if (p.num_seqs == 0) return cudaSuccess;
    const int64_t rows = (int64_t)p.num_blocks * p.num_kv_heads * p.block_size;
    CUtensorMap mk, mv;
    if (!make_cache_tensor_map(&mk, p.k_cache, dtype, p.head_dim, rows, p.block_size) ||
        !make_cache_tensor_map(&mv, p.v_cache, dtype, p.head_dim, rows, p.block_size))
        return cudaErrorInvalidValue;
    if (dtype == PA_BF16)
        return p.head_dim == 128 ? tc::launch_tc_d<__nv_bfloat16, 128>(p, mk, mv, stream)
                                 : tc::launch_tc_d<__nv_bfloat16, 64>(p, mk, mv, stream);
    return p.head_dim == 128 ? tc::launch_tc_d<__half, 128>(p, mk, mv, stream)
                             : tc::launch_tc_d<__half, 64>(p, mk, mv, stream);
}

}  // namespace pa
