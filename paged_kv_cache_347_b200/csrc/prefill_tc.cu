// Causal multi-token attention over the paged cache (chunked prefill), for
// 16-bit caches on sm_100a.
//
// The same quantity as the decode -- attention through the block table,
// keys and values read one block at a time with an online softmax
// (mbrenndoerfer.com "Paged Attention > Summary", bullet 3) -- for several new
// tokens of a sequence at once: row r of the chunk sits at position
// L - n + r and attends to positions 0..L-n+r (paweldubiel.com
// "PagedAttention", "Mechanism and details": the new tokens are appended after
// the prefix, whose blocks stay where they are).
//
// Here the GQA group times the chunk's tokens is a dense tile, so the kernel
// is a FlashAttention-style tensor-core loop:
//
//  * CTA = (tile of T = 64/G chunk tokens, KV head g, sequence s): 64 rows =
//    (token, query head) pairs, 4 consumer warps of 16 rows and 1 producer
//    warp.  The producer streams the keys 0..(last position of the tile) in
//    stages of 64 through a 2-stage ring with TMA tensor loads of each block's
//    K/V rows (128-byte boxes, 128B swizzle, no multicast), as in the decode.
//  * Each consumer warp computes S = Q K^T for its 16 rows and the stage's 64
//    keys (mma.sync m16n8k16, Q fragments held in registers, K via ldmatrix),
//    masks keys after each row's position, updates the running max/sum in
//    fp32, and accumulates O += P V (P from the S accumulators in registers,
//    split into 16-bit high and remainder parts for ~16-bit weights; V via
//    ldmatrix.trans).  Rows are independent, so there is no cross-warp merge.
//
// All waits are bounded as in the decode kernel.
#include <math.h>

#include <mutex>

#include "decode_common.cuh"
#include "prefill_common.cuh"

namespace pa {
namespace pf {

constexpr int kWarps = 4;
constexpr int kThreads = (kWarps + 1) * 32;
constexpr int kRows = 16 * kWarps;  // (token, head) rows per CTA
static_assert(kRows == 64, "the ABI sizes this kernel's grid with 64 / G tokens per CTA");
constexpr int kStageKeys = 64;
constexpr int kRowBytes = 128;

template <typename T, int D, int BS, int NS>
struct Cfg {
    static constexpr int kPieces = D / 64;
    static constexpr int kPieceBytes = kStageKeys * kRowBytes;  // 8 KB
    static constexpr int kKBytes = kPieces * kPieceBytes;
    static constexpr int kStageBytes = 2 * kKBytes;
    static constexpr int kBlocksPerStage = kStageKeys / BS;
    static constexpr int kBarOffset = NS * kStageBytes;
    static constexpr int kAbortOffset = kBarOffset + 2 * NS * 8;
    static constexpr int kSmemBytes = kAbortOffset + 16;
    static constexpr int kDynSmem = kSmemBytes + 1024;
    static_assert(kStageKeys % BS == 0 && kBlocksPerStage <= 32, "block size");
    static_assert(sizeof(T) == 2, "16-bit caches");
};

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

template <typename T, int D, int BS, int NS>
__global__ void __launch_bounds__(kThreads) prefill_tc_kernel(
    const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
    const PrefillParams p) {
    using C = Cfg<T, D, BS, NS>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

    pdl_wait_prior_grid();

    const int qt = blockIdx.x, g = blockIdx.y, s = blockIdx.z;
    const int G = p.num_heads / p.num_kv_heads;
    const int TQ = p.tokens_per_cta;
    const int q0 = __ldg(p.cu_q + s);
    const int n = __ldg(p.cu_q + s + 1) - q0;
    const int L = __ldg(p.seq_lens + s);
    if (n < 0 || n > L || L > p.max_seq_len || n > p.max_q_len ||
        (int64_t)(L + BS - 1) / BS > p.max_blocks_per_seq) {
        if (qt == 0 && g == 0 && threadIdx.x == 0) raise_device_error(p.err, PA_DEVERR_SEQLEN);
        return;
    }
    const int tok0 = qt * TQ;
    if (tok0 >= n) return;  // uniform over the CTA, before any barrier
    const int ntok = min(TQ, n - tok0);
    const int pos0 = L - n + tok0;       // position of the tile's first token
    const int nkeys = pos0 + ntok;       // keys 0 .. last position of the tile
    const int nstages = (nkeys + kStageKeys - 1) / kStageKeys;
    const int nblk = (nkeys + BS - 1) / BS;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::kBarOffset);
    const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + NS);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::kAbortOffset);
    if (threadIdx.x == 0) {
        for (int i = 0; i < NS; ++i) {
            mbar_init(full0 + 8 * i, 1);
            mbar_init(empty0 + 8 * i, kWarps);
        }
        *abort_flag = 0;
        fence_mbarrier_init();
    }
    __syncthreads();
    const uint32_t stage0 = smem_u32(smem);

    // ------------------------------------------------------------ producer
    if (warp == kWarps) {
        if (lane == 0) {
            prefetch_tensormap(&tmap_k);
            prefetch_tensormap(&tmap_v);
        }
        const uint64_t policy = l2_policy_evict_normal();
        int issued = 0;
        for (int i = 0; i < nstages; ++i) {
            // the stage's table entries, one per lane, gathered in lane 0
            const int jb = i * C::kBlocksPerStage;
            const int jn = min(C::kBlocksPerStage, nblk - jb);
            int mine = 0;
            if (lane < jn) {
                const int b = checked_block_row(p.block_tables, p.max_blocks_per_seq, p.num_blocks,
                                                p.err, s, jb + lane);
                mine = b < 0 ? p.num_blocks : b;  // out of range: TMA fills zeros
            }
            int ent[C::kBlocksPerStage];
#pragma unroll
            for (int j = 0; j < C::kBlocksPerStage; ++j) ent[j] = __shfl_sync(0xffffffffu, mine, j);
            int stop = 0;
            if (lane == 0) {
                const int buf = i % NS;
                if (i >= NS &&
                    !mbar_wait_bounded(empty0 + 8 * buf, ((i / NS) - 1) & 1, abort_flag)) {
                    raise_device_error(p.err, PA_DEVERR_TIMEOUT);
                    *abort_flag = 1;
                    stop = 1;
                } else {
                    const uint32_t full = full0 + 8 * buf;
                    mbar_arrive_expect_tx(full, (uint32_t)(jn * 4 * BS * D));
                    const uint32_t kdst = stage0 + buf * C::kStageBytes;
                    const uint32_t vdst = kdst + C::kKBytes;
#pragma unroll
                    for (int j = 0; j < C::kBlocksPerStage; ++j) {
                        if (j < jn) {
                            const int y = (ent[j] * p.num_kv_heads + g) * BS;
#pragma unroll
                            for (int pc = 0; pc < C::kPieces; ++pc) {
                                const uint32_t off = pc * C::kPieceBytes + j * BS * kRowBytes;
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
        if (lane == 0) {
            for (int i = max(0, issued - NS); i < issued; ++i)
                mbar_wait_bounded(full0 + 8 * (i % NS), (i / NS) & 1, nullptr);
        }
        return;
    }

    // ------------------------------------------------------------ consumers
    const int gid = lane >> 2, tig = lane & 3;
    // rows gid and gid + 8 of this warp: (token, head) = (r / G, r % G)
    const int r_lo = 16 * warp + gid, r_hi = r_lo + 8;
    const int t_lo = r_lo / G, t_hi = r_hi / G;
    const bool v_lo = t_lo < ntok && r_lo < TQ * G, v_hi = t_hi < ntok && r_hi < TQ * G;
    // positions; rows that do not exist attend to every key (kept finite)
    const int qp_lo = v_lo ? pos0 + t_lo : nkeys - 1;
    const int qp_hi = v_hi ? pos0 + t_hi : nkeys - 1;
    const T *qbase = static_cast<const T *>(p.q);
    const int64_t qrow_lo = ((int64_t)(q0 + tok0 + t_lo) * p.num_heads + g * G + r_lo % G) * D;
    const int64_t qrow_hi = ((int64_t)(q0 + tok0 + t_hi) * p.num_heads + g * G + r_hi % G) * D;
    uint32_t qa[D / 16][4];
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
        const int c = 16 * kk + 2 * tig;
        qa[kk][0] = v_lo ? __ldg(reinterpret_cast<const uint32_t *>(qbase + qrow_lo + c)) : 0u;
        qa[kk][1] = v_hi ? __ldg(reinterpret_cast<const uint32_t *>(qbase + qrow_hi + c)) : 0u;
        qa[kk][2] = v_lo ? __ldg(reinterpret_cast<const uint32_t *>(qbase + qrow_lo + c + 8)) : 0u;
        qa[kk][3] = v_hi ? __ldg(reinterpret_cast<const uint32_t *>(qbase + qrow_hi + c + 8)) : 0u;
    }

    float o[D / 8][4];
#pragma unroll
    for (int nt = 0; nt < D / 8; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;
    float m_lo = -INFINITY, m_hi = -INFINITY, l_lo = 0.f, l_hi = 0.f;
    const float sl2 = p.scale_log2;
    const int r7 = lane & 7;
    const int krow = r7 + ((lane >> 4) << 3);        // key row within a 16-key group (QK)
    const int kchk = (lane >> 3) & 1;
    const int vrow = r7 + (((lane >> 3) & 1) << 3);  // key row within a 16-key group (PV)
    const int vchk = lane >> 4;
    bool ok = true;

    for (int i = 0; i < nstages; ++i) {
        const int buf = i % NS;
        if (!warp_wait(full0 + 8 * buf, (i / NS) & 1, abort_flag, lane)) {
            ok = false;
            break;
        }
        const uint32_t kbase = stage0 + buf * C::kStageBytes;
        const uint32_t vbase = kbase + C::kKBytes;
        const int kb = i * kStageKeys;
        // ---- S = Q K^T: 8 n-tiles of 8 keys
        float sc[8][4];
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
            for (int np = 0; np < 4; ++np) {
                const int row = 16 * np + krow;
                const int chunk = ((kk & 3) << 1) + kchk;
                const uint32_t addr = kbase + (kk >> 2) * C::kPieceBytes + row * kRowBytes +
                                      ((chunk ^ r7) << 4);
                uint32_t b[4];
                ldmatrix_x4(addr, b[0], b[1], b[2], b[3]);
                Mma<T>::run(sc[2 * np], qa[kk], b[0], b[1]);
                Mma<T>::run(sc[2 * np + 1], qa[kk], b[2], b[3]);
            }
        }
        // ---- causal mask, online softmax (log2 domain)
        const bool need_mask = kb + kStageKeys - 1 > pos0;
        float mx_lo = -INFINITY, mx_hi = -INFINITY;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
            const int key = kb + 8 * nt + 2 * tig;
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                float xl = sc[nt][e] * sl2, xh = sc[nt][2 + e] * sl2;
                if (need_mask) {
                    if (key + e > qp_lo) xl = -INFINITY;
                    if (key + e > qp_hi) xh = -INFINITY;
                }
                sc[nt][e] = xl;
                sc[nt][2 + e] = xh;
                mx_lo = fmaxf(mx_lo, xl);
                mx_hi = fmaxf(mx_hi, xh);
            }
        }
#pragma unroll
        for (int off = 1; off < 4; off <<= 1) {
            mx_lo = fmaxf(mx_lo, __shfl_xor_sync(0xffffffffu, mx_lo, off));
            mx_hi = fmaxf(mx_hi, __shfl_xor_sync(0xffffffffu, mx_hi, off));
        }
        // every row has key 0 in stage 0, so the running max is finite from there on
        const float mn_lo = fmaxf(m_lo, mx_lo), mn_hi = fmaxf(m_hi, mx_hi);
        const float al_lo = exp2f(m_lo - mn_lo), al_hi = exp2f(m_hi - mn_hi);
        m_lo = mn_lo;
        m_hi = mn_hi;
        float sum_lo = 0.f, sum_hi = 0.f;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
            sc[nt][0] = exp2f(sc[nt][0] - mn_lo);
            sc[nt][1] = exp2f(sc[nt][1] - mn_lo);
            sc[nt][2] = exp2f(sc[nt][2] - mn_hi);
            sc[nt][3] = exp2f(sc[nt][3] - mn_hi);
            sum_lo += sc[nt][0] + sc[nt][1];
            sum_hi += sc[nt][2] + sc[nt][3];
        }
        l_lo = l_lo * al_lo + sum_lo;
        l_hi = l_hi * al_hi + sum_hi;
#pragma unroll
        for (int nt = 0; nt < D / 8; ++nt) {
            o[nt][0] *= al_lo;
            o[nt][1] *= al_lo;
            o[nt][2] *= al_hi;
            o[nt][3] *= al_hi;
        }
        // keys past the tile's last position may be stale rows: zero their V
        const bool tail = kb + kStageKeys > nkeys;
        // ---- O += P V, 4 k-steps of 16 keys
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            uint32_t ph[4], pl[4];
            ph[0] = Mma<T>::pack(sc[2 * j][0], sc[2 * j][1]);
            ph[1] = Mma<T>::pack(sc[2 * j][2], sc[2 * j][3]);
            ph[2] = Mma<T>::pack(sc[2 * j + 1][0], sc[2 * j + 1][1]);
            ph[3] = Mma<T>::pack(sc[2 * j + 1][2], sc[2 * j + 1][3]);
            pl[0] = Mma<T>::pack(sc[2 * j][0] - Mma<T>::lo(ph[0]), sc[2 * j][1] - Mma<T>::hi(ph[0]));
            pl[1] = Mma<T>::pack(sc[2 * j][2] - Mma<T>::lo(ph[1]), sc[2 * j][3] - Mma<T>::hi(ph[1]));
            pl[2] = Mma<T>::pack(sc[2 * j + 1][0] - Mma<T>::lo(ph[2]),
                                 sc[2 * j + 1][1] - Mma<T>::hi(ph[2]));
            pl[3] = Mma<T>::pack(sc[2 * j + 1][2] - Mma<T>::lo(ph[3]),
                                 sc[2 * j + 1][3] - Mma<T>::hi(ph[3]));
            uint32_t vm0 = 0xffffffffu, vm1 = 0xffffffffu;
            if (tail) {
                const int k0 = kb + 16 * j + 2 * tig;
                vm0 = (k0 < nkeys ? 0x0000ffffu : 0u) | (k0 + 1 < nkeys ? 0xffff0000u : 0u);
                vm1 = (k0 + 8 < nkeys ? 0x0000ffffu : 0u) | (k0 + 9 < nkeys ? 0xffff0000u : 0u);
            }
#pragma unroll
            for (int dp = 0; dp < D / 16; ++dp) {
                const int row = 16 * j + vrow;
                const int d0 = 16 * dp + 8 * vchk;
                const int chunk = (d0 & 63) >> 3;
                const uint32_t addr = vbase + (d0 >> 6) * C::kPieceBytes + row * kRowBytes +
                                      ((chunk ^ r7) << 4);
                uint32_t b[4];
                ldmatrix_x4_trans(addr, b[0], b[1], b[2], b[3]);
                b[0] &= vm0;
                b[1] &= vm1;
                b[2] &= vm0;
                b[3] &= vm1;
                Mma<T>::run(o[2 * dp], ph, b[0], b[1]);
                Mma<T>::run(o[2 * dp], pl, b[0], b[1]);
                Mma<T>::run(o[2 * dp + 1], ph, b[2], b[3]);
                Mma<T>::run(o[2 * dp + 1], pl, b[2], b[3]);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty0 + 8 * buf);
    }
    if (!ok) {
        if (lane == 0) {
            raise_device_error(p.err, PA_DEVERR_TIMEOUT);
            *abort_flag = 1;
        }
        return;
    }

    // ------------------------------------------------------------ store
#pragma unroll
    for (int off = 1; off < 4; off <<= 1) {
        l_lo += __shfl_xor_sync(0xffffffffu, l_lo, off);
        l_hi += __shfl_xor_sync(0xffffffffu, l_hi, off);
    }
    const float inv_lo = l_lo > 0.f ? 1.f / l_lo : 0.f;
    const float inv_hi = l_hi > 0.f ? 1.f / l_hi : 0.f;
    float *out_lo = p.out + qrow_lo, *out_hi = p.out + qrow_hi;
#pragma unroll
    for (int nt = 0; nt < D / 8; ++nt) {
        const int d = 8 * nt + 2 * tig;
        if (v_lo) *reinterpret_cast<float2 *>(out_lo + d) = make_float2(o[nt][0] * inv_lo, o[nt][1] * inv_lo);
        if (v_hi) *reinterpret_cast<float2 *>(out_hi + d) = make_float2(o[nt][2] * inv_hi, o[nt][3] * inv_hi);
    }
}

template <typename T, int D, int BS>
static cudaError_t launch_inst(const PrefillParams &p, const CUtensorMap &mk,
                               const CUtensorMap &mv, cudaStream_t stream) {
    constexpr int NS = 2;
    using C = Cfg<T, D, BS, NS>;
    static std::once_flag once[64];
    static cudaError_t attr_err[64];
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::call_once(once[dev], [&] {
        attr_err[dev] = cudaFuncSetAttribute(prefill_tc_kernel<T, D, BS, NS>,
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
    return cudaLaunchKernelEx(&cfg, prefill_tc_kernel<T, D, BS, NS>, mk, mv, p);
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

}  // namespace pf

cudaError_t launch_prefill_tc(const PrefillParams &p, int dtype, cudaStream_t stream) {
    if (p.num_seqs == 0 || p.max_q_len == 0) return cudaSuccess;
    const int64_t rows = (int64_t)p.num_blocks * p.num_kv_heads * p.block_size;
    CUtensorMap mk, mv;
    if (!make_cache_tensor_map(&mk, p.k_cache, dtype, p.head_dim, rows, p.block_size) ||
        !make_cache_tensor_map(&mv, p.v_cache, dtype, p.head_dim, rows, p.block_size))
        return cudaErrorInvalidValue;
    if (dtype == PA_BF16)
        return p.head_dim == 128 ? pf::launch_d<__nv_bfloat16, 128>(p, mk, mv, stream)
                                 : pf::launch_d<__nv_bfloat16, 64>(p, mk, mv, stream);
    return p.head_dim == 128 ? pf::launch_d<__half, 128>(p, mk, mv, stream)
                             : pf::launch_d<__half, 64>(p, mk, mv, stream);
}

}  // namespace pa
