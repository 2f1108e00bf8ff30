// Causal multi-token attention over the paged cache on the 5th-generation
// tensor cores (tcgen05, accumulators in TMEM), sm_100a.
//
// Same quantity as prefill_tc.cu (mbrenndoerfer.com "Paged Attention >
// Summary", bullet 3; paweldubiel.com "PagedAttention", "Mechanism and
// details"): row r of a sequence's chunk, at position L - n + r, attends to
// positions 0..L-n+r through the block table.
//
// CTA = 128 (token, query head) rows: 128/G chunk tokens of one KV head g of
// one sequence.  Six warps:
//   * warps 0-3 (one thread per row, thread i <-> TMEM lane i): load the Q rows
//     into a 128B-swizzled shared tile; per stage read the S tile from TMEM,
//     apply the causal mask, keep the row's running max and sum in fp32, write
//     P (bf16/f16 high part and remainder) into a swizzled shared tile,
//     rescale the O accumulator in TMEM when the row max grows by more than
//     2^8; at the end read O from TMEM, divide by the sum and store;
//   * warp 4: TMA producer of 64-key K/V stages (the decode's ring);
//   * warp 5, one thread: issues the UMMAs --
//       S[128 x 64]  = Q[128 x D] . K_stage^T            (both K-major)
//       O[128 x D]  += P[128 x 64] . V_stage[64 x D]     (P K-major, V N-major)
//     and commits them to mbarriers.  S is double-buffered in TMEM, so S of
//     stage i+1 is computed while the softmax works on stage i.
// TMEM: S0 (64 cols), S1 (64), O (D): 256 columns allocated.
//
// Every wait is bounded (~2 s); on a timeout the CTA records
// PA_DEVERR_TIMEOUT, waits (bounded) for its own copies and MMAs, frees its
// TMEM and exits.
#include <math.h>

#include <mutex>

#include "decode_common.cuh"
#include "umma.cuh"

namespace pa {
namespace pu {

constexpr int kM = 128;          // rows per CTA
constexpr int kKeys = 64;        // keys per stage
constexpr int kThreads = 6 * 32;
constexpr int kSoftmaxThreads = 128;
constexpr int kTmemCols = 256;
constexpr int kRowBytes = 128;

template <int D, int BS, int NS>
struct Cfg {
    static constexpr int kPieces = D / 64;
    static constexpr int kQPiece = kM * kRowBytes;              // 16 KB
    static constexpr int kQBytes = kPieces * kQPiece;
    static constexpr int kKVPiece = kKeys * kRowBytes;          // 8 KB
    static constexpr int kKBytes = kPieces * kKVPiece;
    static constexpr int kStageBytes = 2 * kKBytes;             // K + V
    static constexpr int kPTile = kM * kRowBytes;               // 128 rows x 64 keys x 2 B
    static constexpr int kPBytes = 2 * kPTile;                  // high part + remainder
    static constexpr int kQOffset = 0;
    static constexpr int kKVOffset = kQBytes;
    static constexpr int kPOffset = kKVOffset + NS * kStageBytes;
    static constexpr int kBarOffset = kPOffset + 2 * kPBytes;
    // barriers: kv_full[NS] kv_empty[NS] s_full[2] s_empty[2] p_full[2] pv_done[2] q_full mma_done
    static constexpr int kNumBars = 2 * NS + 8 + 2;
    static constexpr int kTmemSlot = kBarOffset + kNumBars * 8;
    static constexpr int kAbortOffset = kTmemSlot + 16;
    static constexpr int kSmemBytes = kAbortOffset + 16;
    static constexpr int kDynSmem = kSmemBytes + 1024;
    static constexpr int kBlocksPerStage = kKeys / BS;
    static_assert(kDynSmem <= 227 * 1024, "shared memory");
    static_assert(kKeys % BS == 0, "block size divides a stage");
};

__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int *abort_flag) {
    return mbar_wait_bounded(bar, parity, abort_flag);
}

// The same wait taken by a whole warp, with one outcome for all its lanes
// (the tcgen05 loads and stores that follow are warp-collective).
__device__ __forceinline__ bool warp_wait_bar(uint32_t bar, uint32_t parity,
                                              volatile int *abort_flag) {
    return __all_sync(0xffffffffu, mbar_wait_bounded(bar, parity, abort_flag));
}

template <typename T, int D, int BS, int NS>
__global__ void __launch_bounds__(kThreads, 1) prefill_umma_kernel(
    const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
    const PrefillParams p) {
    using C = Cfg<D, BS, NS>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

    pdl_wait_prior_grid();

    const int qt = blockIdx.x, g = blockIdx.y, s = blockIdx.z;
    const int G = p.num_heads / p.num_kv_heads;
    const int TQ = p.tokens_per_cta;  // 128 / G
    const int q0 = __ldg(p.cu_q + s);
    const int n = __ldg(p.cu_q + s + 1) - q0;
    const int L = __ldg(p.seq_lens + s);
    if (n < 0 || n > L || L > p.max_seq_len || n > p.max_q_len ||
        (int64_t)(L + BS - 1) / BS > p.max_blocks_per_seq) {
        if (qt == 0 && g == 0 && threadIdx.x == 0) raise_device_error(p.err, PA_DEVERR_SEQLEN);
        return;
    }
    const int tok0 = qt * TQ;
    if (tok0 >= n) return;  // uniform, before any barrier or TMEM use
    const int ntok = min(TQ, n - tok0);
    const int pos0 = L - n + tok0;
    const int nkeys = pos0 + ntok;
    const int nstages = (nkeys + kKeys - 1) / kKeys;
    const int nblk = (nkeys + BS - 1) / BS;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    const uint32_t sbase = smem_u32(smem);
    const uint32_t q_s = sbase + C::kQOffset, kv_s = sbase + C::kKVOffset, p_s = sbase + C::kPOffset;
    const uint32_t bar0 = sbase + C::kBarOffset;
    const uint32_t kv_full = bar0, kv_empty = bar0 + 8 * NS, s_full = bar0 + 16 * NS,
                   s_empty = s_full + 16, p_full = s_empty + 16, pv_done = p_full + 16,
                   q_full = pv_done + 16, mma_done = q_full + 8;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::kAbortOffset);
    volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(smem + C::kTmemSlot);

    if (threadIdx.x == 0) {
        for (int i = 0; i < NS; ++i) {
            mbar_init(kv_full + 8 * i, 1);
            mbar_init(kv_empty + 8 * i, 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(s_full + 8 * i, 1);
            mbar_init(s_empty + 8 * i, kSoftmaxThreads);
            mbar_init(p_full + 8 * i, kSoftmaxThreads);
            mbar_init(pv_done + 8 * i, 1);
        }
        mbar_init(q_full, kSoftmaxThreads);
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        fence_mbarrier_init();
    }
    if (warp == 0) {
        umma::tmem_alloc(sbase + C::kTmemSlot, kTmemCols);
        umma::tmem_relinquish();
    }
    umma::fence_before_sync();
    __syncthreads();
    umma::fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    // ------------------------------------------------------------ producer
    if (warp == 4) {
        if (lane == 0) {
            prefetch_tensormap(&tmap_k);
            prefetch_tensormap(&tmap_v);
        }
        const uint64_t policy = l2_policy_evict_first();
        int issued = 0;
        for (int i = 0; i < nstages; ++i) {
            const int jb = i * C::kBlocksPerStage;
            const int jn = min(C::kBlocksPerStage, nblk - jb);
            int mine = 0;
            if (lane < jn) {
                const int b = checked_block_row(p.block_tables, p.max_blocks_per_seq, p.num_blocks,
                                                p.err, s, jb + lane);
                mine = b < 0 ? p.num_blocks : b;
            }
            int ent[C::kBlocksPerStage];
#pragma unroll
            for (int j = 0; j < C::kBlocksPerStage; ++j) ent[j] = __shfl_sync(0xffffffffu, mine, j);
            int stop = 0;
            if (lane == 0) {
                const int buf = i % NS;
                if (i >= NS && !wait_bar(kv_empty + 8 * buf, ((i / NS) - 1) & 1, abort_flag)) {
                    raise_device_error(p.err, PA_DEVERR_TIMEOUT);
                    *abort_flag = 1;
                    stop = 1;
                } else {
                    const uint32_t full = kv_full + 8 * buf;
                    mbar_arrive_expect_tx(full, (uint32_t)(jn * 4 * BS * D));
                    const uint32_t kdst = kv_s + buf * C::kStageBytes;
                    const uint32_t vdst = kdst + C::kKBytes;
#pragma unroll
                    for (int j = 0; j < C::kBlocksPerStage; ++j) {
                        if (j < jn) {
                            const int y = (ent[j] * p.num_kv_heads + g) * BS;
#pragma unroll
                            for (int pc = 0; pc < C::kPieces; ++pc) {
                                const uint32_t off = pc * C::kKVPiece + j * BS * kRowBytes;
                                tma_load_2d(kdst + off, &tmap_k, pc * 64, y, full, policy);
                                tma_load_2d(vdst + off, &tmap_v, pc * 64, y, full, policy);
                            }
                        }
                    }
                    issued = i + 1;
                }
            }
            if (__shfl_sync(0xffffffffu, stop, 0)) break;
        }
        if (lane == 0)
            for (int i = max(0, issued - NS); i < issued; ++i)
                mbar_wait_bounded(kv_full + 8 * (i % NS), (i / NS) & 1, nullptr);
        return;
    }

    // ------------------------------------------------------------ MMA issuer
    if (warp == 5) {
        if (lane == 0) {
            constexpr uint32_t fmt = StoreT<T>::kCode == PA_BF16 ? 1u : 0u;
            constexpr uint32_t idesc_s = umma::idesc_f16(fmt, kM, kKeys, 0);
            constexpr uint32_t idesc_o = umma::idesc_f16(fmt, kM, D, 1);
            bool ok = wait_bar(q_full, 0, abort_flag);
            // S_i = Q . K_i^T into TMEM columns 64 * (i % 2)
            auto issue_s = [&](int i) -> bool {
                const int buf = i % NS;
                if (!wait_bar(kv_full + 8 * buf, (i / NS) & 1, abort_flag)) return false;
                if (i >= 2 && !wait_bar(s_empty + 8 * (i % 2), ((i / 2) - 1) & 1, abort_flag))
                    return false;
                umma::fence_after_sync();
                const uint32_t kst = kv_s + buf * C::kStageBytes;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t a = umma::smem_desc_sw128(
                        q_s + (kk >> 2) * C::kQPiece + (kk & 3) * 32, 16, 1024);
                    const uint64_t b = umma::smem_desc_sw128(
                        kst + (kk >> 2) * C::kKVPiece + (kk & 3) * 32, 16, 1024);
                    umma::mma_f16(tmem + (i % 2) * kKeys, a, b, idesc_s, kk > 0);
                }
                umma::commit(s_full + 8 * (i % 2));
                return true;
            };
            if (ok) ok = issue_s(0);
            for (int i = 0; ok && i < nstages; ++i) {
                if (i + 1 < nstages && !issue_s(i + 1)) {
                    ok = false;
                    break;
                }
                // O += P_i . V_i once the softmax has written P_i
                if (!wait_bar(p_full + 8 * (i % 2), (i / 2) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                umma::fence_after_sync();
                const uint32_t vst = kv_s + (i % NS) * C::kStageBytes + C::kKBytes;
                const uint32_t pst = p_s + (i % 2) * C::kPBytes;
#pragma unroll
                for (int j = 0; j < kKeys / 16; ++j) {
                    const uint64_t b = umma::smem_desc_sw128(vst + j * 16 * kRowBytes,
                                                             C::kKVPiece, 1024);
                    const uint64_t a_hi = umma::smem_desc_sw128(pst + j * 32, 16, 1024);
                    const uint64_t a_lo = umma::smem_desc_sw128(pst + C::kPTile + j * 32, 16, 1024);
                    umma::mma_f16(tmem + 2 * kKeys, a_hi, b, idesc_o, (i > 0 || j > 0) ? 1u : 0u);
                    umma::mma_f16(tmem + 2 * kKeys, a_lo, b, idesc_o, 1u);
                }
                umma::commit(pv_done + 8 * (i % 2));
                umma::commit(kv_empty + 8 * (i % NS));
            }
            if (!ok) {
                raise_device_error(p.err, PA_DEVERR_TIMEOUT);
                *abort_flag = 1;
            }
            umma::commit(mma_done);  // arrives when every MMA issued above is done
        }
        return;
    }

    // ------------------------------------------------------------ softmax warps
    const int r = threadIdx.x;  // row == TMEM lane
    const int t = r / G, hh = r - (r / G) * G;
    const bool valid = t < ntok && r < TQ * G;
    const int qp = valid ? pos0 + t : nkeys - 1;
    const int64_t qrow = ((int64_t)(q0 + tok0 + t) * p.num_heads + g * G + hh) * D;
    {
        // Q row -> swizzled K-major tile (row r, 16-byte chunk c at c ^ (r & 7))
        const uint4 *src = reinterpret_cast<const uint4 *>(static_cast<const T *>(p.q) + qrow);
#pragma unroll
        for (int c = 0; c < D / 8; ++c) {
            const uint4 v = valid ? __ldg(src + c) : make_uint4(0u, 0u, 0u, 0u);
            const int pc = c >> 3, cc = c & 7;
            *reinterpret_cast<uint4 *>(smem + C::kQOffset + pc * C::kQPiece + r * kRowBytes +
                                       ((cc ^ (r & 7)) << 4)) = v;
        }
        umma::fence_proxy_async_smem();
        mbar_arrive(q_full);
    }
    const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
    const float sl2 = p.scale_log2;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int i = 0; i < nstages; ++i) {
        const int sb = i % 2;
        if (!warp_wait_bar(s_full + 8 * sb, (i / 2) & 1, abort_flag)) {
            ok = false;
            break;
        }
        umma::fence_after_sync();
        uint32_t sr[2][32];
        umma::ld32(lane_base + sb * kKeys, sr[0]);
        umma::ld32(lane_base + sb * kKeys + 32, sr[1]);
        umma::wait_ld();
        umma::fence_before_sync();
        mbar_arrive(s_empty + 8 * sb);
        const int kb = i * kKeys;
        float x[kKeys];
        float mx = -INFINITY;
#pragma unroll
        for (int c = 0; c < kKeys; ++c) {
            const float v = __uint_as_float(sr[c >> 5][c & 31]) * sl2;
            x[c] = kb + c > qp ? -INFINITY : v;
            mx = fmaxf(mx, x[c]);
        }
        // the running max moves only when it grows by more than 8 (log2 units):
        // weights then stay below 2^8 and O is rescaled rarely
        float alpha = 1.f;
        bool rescale = false;
        if (mx > m + 8.f) {
            alpha = exp2f(m - mx);  // 0 on the first stage (m = -inf)
            rescale = m != -INFINITY;
            m = mx;
        }
        float sum = 0.f;
#pragma unroll
        for (int c = 0; c < kKeys; ++c) {
            x[c] = exp2f(x[c] - m);
            sum += x[c];
        }
        l = l * alpha + sum;
        // PV of stage i-1 (and of i-2, which used this P buffer) must be done
        if (i > 0 && !warp_wait_bar(pv_done + 8 * ((i - 1) % 2), ((i - 1) / 2) & 1, abort_flag)) {
            ok = false;
            break;
        }
        if (__any_sync(0xffffffffu, rescale)) {  // warp-collective TMEM access
            umma::fence_after_sync();
#pragma unroll
            for (int cb = 0; cb < D / 32; ++cb) {
                uint32_t orr[32];
                umma::ld32(lane_base + 2 * kKeys + cb * 32, orr);
                umma::wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) orr[e] = __float_as_uint(__uint_as_float(orr[e]) * alpha);
                umma::st32(lane_base + 2 * kKeys + cb * 32, orr);
            }
            umma::wait_st();
        }
        // stale K/V rows past the last key of the tile: zero V so 0 * x stays 0
        if (kb + kKeys > nkeys) {
            // the stage's copies have landed (the S MMA waited for them); this
            // wait only orders the zero stores after them
            if (!warp_wait_bar(kv_full + 8 * (i % NS), (i / NS) & 1, abort_flag)) {
                ok = false;
                break;
            }
            const int first = nkeys - kb;  // rows [first, 64) of this stage
            uint8_t *vst = smem + C::kKVOffset + (i % NS) * C::kStageBytes + C::kKBytes;
            for (int idx = r; idx < (kKeys - first) * C::kPieces * 8; idx += kSoftmaxThreads) {
                const int row = first + idx / (C::kPieces * 8);
                const int rem = idx % (C::kPieces * 8);
                *reinterpret_cast<uint4 *>(vst + (rem >> 3) * C::kKVPiece + row * kRowBytes +
                                           ((rem & 7) << 4)) = make_uint4(0u, 0u, 0u, 0u);
            }
        }
        // P (high part, remainder) -> swizzled K-major tiles, row r
        uint8_t *ph = smem + C::kPOffset + sb * C::kPBytes;
#pragma unroll
        for (int c = 0; c < kKeys / 8; ++c) {
            uint32_t hi[4], lo[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                hi[e] = Mma<T>::pack(x[8 * c + 2 * e], x[8 * c + 2 * e + 1]);
                lo[e] = Mma<T>::pack(x[8 * c + 2 * e] - Mma<T>::lo(hi[e]),
                                     x[8 * c + 2 * e + 1] - Mma<T>::hi(hi[e]));
            }
            const int off = r * kRowBytes + ((c ^ (r & 7)) << 4);
            *reinterpret_cast<uint4 *>(ph + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
            *reinterpret_cast<uint4 *>(ph + C::kPTile + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        }
        umma::fence_proxy_async_smem();
        umma::fence_before_sync();
        mbar_arrive(p_full + 8 * sb);
    }
    if (ok && !warp_wait_bar(pv_done + 8 * ((nstages - 1) % 2), ((nstages - 1) / 2) & 1, abort_flag))
        ok = false;
    if (ok) {
        umma::fence_after_sync();
        const float inv = l > 0.f ? 1.f / l : 0.f;
        float *dst = p.out + qrow;
#pragma unroll
        for (int cb = 0; cb < D / 32; ++cb) {
            uint32_t orr[32];
            umma::ld32(lane_base + 2 * kKeys + cb * 32, orr);
            umma::wait_ld();
            if (valid) {
#pragma unroll
                for (int e = 0; e < 32; e += 4)
                    *reinterpret_cast<float4 *>(dst + cb * 32 + e) =
                        make_float4(__uint_as_float(orr[e]) * inv, __uint_as_float(orr[e + 1]) * inv,
                                    __uint_as_float(orr[e + 2]) * inv,
                                    __uint_as_float(orr[e + 3]) * inv);
            }
        }
    } else if (lane == 0) {
        raise_device_error(p.err, PA_DEVERR_TIMEOUT);
        *abort_flag = 1;  // the other warps stop waiting
    }
    // TMEM is freed once every MMA of this CTA has completed and every
    // softmax warp is done reading it
    umma::fence_before_sync();
    named_barrier_sync(1, kSoftmaxThreads);
    if (warp == 0) {
        mbar_wait_bounded(mma_done, 0, nullptr);
        umma::fence_after_sync();
        umma::tmem_dealloc(tmem, kTmemCols);
    }
    pdl_launch_dependents();
}

template <typename T, int D, int BS>
static cudaError_t launch_inst(const PrefillParams &p, const CUtensorMap &mk,
                               const CUtensorMap &mv, cudaStream_t stream) {
    constexpr int NS = 2;
    using C = Cfg<D, BS, NS>;
    static std::once_flag once[64];
    static cudaError_t attr_err[64];
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::call_once(once[dev], [&] {
        attr_err[dev] = cudaFuncSetAttribute(prefill_umma_kernel<T, D, BS, NS>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             C::kDynSmem);
    });
    if (attr_err[dev] != cudaSuccess) return attr_err[dev];
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((p.max_q_len + p.tokens_per_cta - 1) / p.tokens_per_cta, p.num_kv_heads,
                       p.num_seqs);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = C::kDynSmem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, prefill_umma_kernel<T, D, BS, NS>, mk, mv, p);
}

template <typename T, int D>
static cudaError_t launch_d(const PrefillParams &p, const CUtensorMap &mk, const CUtensorMap &mv,
                            cudaStream_t stream) {
    switch (p.block_size) {
    case 8: return launch_inst<T, D, 8>(p, mk, mv, stream);
    case 16: return launch_inst<T, D, 16>(p, mk, mv, stream);
    case 32: return launch_inst<T, D, 32>(p, mk, mv, stream);
    case 64: return launch_inst<T, D, 64>(p, mk, mv, stream);
    default: return cudaErrorNotSupported;
    }
}

}  // namespace pu

cudaError_t launch_prefill_umma(const PrefillParams &p, int dtype, cudaStream_t stream) {
    if (p.num_seqs == 0 || p.max_q_len == 0) return cudaSuccess;
    const int64_t rows = (int64_t)p.num_blocks * p.num_kv_heads * p.block_size;
    CUtensorMap mk, mv;
    if (!make_cache_tensor_map(&mk, p.k_cache, dtype, p.head_dim, rows, p.block_size) ||
        !make_cache_tensor_map(&mv, p.v_cache, dtype, p.head_dim, rows, p.block_size))
        return cudaErrorInvalidValue;
    if (dtype == PA_BF16)
        return p.head_dim == 128 ? pu::launch_d<__nv_bfloat16, 128>(p, mk, mv, stream)
                                 : pu::launch_d<__nv_bfloat16, 64>(p, mk, mv, stream);
    return p.head_dim == 128 ? pu::launch_d<__half, 128>(p, mk, mv, stream)
                             : pu::launch_d<__half, 64>(p, mk, mv, stream);
}

}  // namespace pa
