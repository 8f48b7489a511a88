// proj.cu -- the projections around the operator, on the tensor cores.
//
// HyenaDNA operator walk-through (adg.csdn.net), section 二.1, HyenaOperator:
//   in_proj  = nn.Linear(d_model, (order+1) d_model) on u [b, l, d], then
//              rearrange 'b l d -> b d l'  (the layout hyena_gated_fftconv reads)
//   out_proj = nn.Linear(d_model, d_model) on rearrange(y, 'b d l -> b l d')
// nn.Linear(x) = x W^T + bias with the weight stored W[out][in].
//
// Both are one batched bf16 GEMM C[M x N] = A[M x K] . B[N x K]^T + bias with
// fp32 accumulation:
//   in_proj : per batch b, M = (order+1) D (output channels), N = L, K = D;
//             A = W_in (K-major), B = x[b] (K-major: D contiguous per position),
//             C = u[b] row-major [M][L]: the rearrangement is the choice of M/N.
//   out_proj: per batch b, M = L, N = D, K = D; A = y[b]^T read in place from
//             y[b] [D][L] (MN-major: positions contiguous), B = W_out (K-major),
//             C = out[b] row-major [L][D].
//
// Kernel: persistent, one CTA per SM, 192 threads in three roles:
//   warp 0   loads A and B tiles (128 x 64 and BN x 64 bf16, 128-byte swizzle)
//            with TMA (cp.async.bulk.tensor, no multicast) into a ring of
//            kStages stages, each completing on a "full" mbarrier;
//   warp 1   issues tcgen05.mma (M 128, N BN, K 16; four per 64-wide K block)
//            into one of two BN-column tensor-memory accumulators, frees each
//            stage with tcgen05.commit to its "empty" mbarrier, and signals a
//            finished tile with a commit to "acc_full";
//   warps 2-5 (the epilogue) read the accumulator rows with tcgen05.ld, add the
//            bias, round to bf16 and store; then free the accumulator
//            ("acc_empty"), so the next tile's MMAs overlap this epilogue.
// Every wait is bounded by a global-time budget; a wait that runs out records
// kStatusTimeout in the device's status word and that role stops issuing work.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <mutex>
#include <string>

#include "hyena.h"
#include "kernels.h"
#include "tc_util.cuh"

namespace hyena {

hyena_status_t set_last_error_detail(hyena_status_t st, const std::string& detail);  // api.cu

namespace {

using bf16 = __nv_bfloat16;

constexpr int BM = 128, BK = 64;
constexpr uint32_t kATile = BM * BK * 2;          // 16 KB
constexpr int kThreadsG = 192;
// Epilogue staging: per epilogue warp 32 rows x 64 columns of bf16, rows
// 144 bytes apart (128 + 16), so that a thread writing its row's 16-byte
// chunks and a warp reading 4 rows x 128 contiguous bytes are both free of
// bank conflicts.
constexpr uint32_t kEpiRow = 144;
constexpr uint32_t kEpiWarp = 32 * kEpiRow;
constexpr uint32_t kEpiBytes = 4 * kEpiWarp;

// Tile width BN (256; 192 or 128 when the wider tiles would leave the grid
// with few waves): B tile, stage size, ring depth, tensor-memory columns (two
// accumulators of BN fp32 columns, allocated as a power of two) and shared
// memory (1024-byte aligned stages, then the barriers).
template <int BN>
struct Cfg {
    static constexpr int kStages = BN == 256 ? 4 : (BN == 192 ? 5 : 6);
    static constexpr uint32_t kBTile = BN * BK * 2;
    static constexpr uint32_t kStageBytes = kATile + kBTile;
    static constexpr uint32_t kAccCols = BN;
    static constexpr uint32_t kTmemCols = 2 * BN <= 256 ? 256 : 512;     // a power of two
    static constexpr size_t kSmem = 1024 + size_t(kStages) * kStageBytes + 256 + (BN == 256 ? kEpiBytes : 0);
};

struct GemmParams {
    int64_t M, N, K, batches;
    int64_t tiles_m, tiles_n;
    int a_mn_major;                 // A read MN-major (out_proj)
    int a_batched, b_batched;       // whether the A / B tensor maps have a batch coordinate
    bf16* c;                        // C[b][m][n] at c + b * c_bstride + m * ldc + n
    int64_t ldc, c_bstride;
    const float* bias;              // [M] (bias_per_row) or [N], or nullptr
    int bias_per_row;
    uint64_t budget_ns;
    uint32_t* status;
};

// UMMA shared-memory descriptor, 128-byte swizzle (layout type 2), sm_100 version.
__device__ __forceinline__ uint64_t desc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= uint64_t((saddr >> 4) & 0x3FFFu);
    d |= uint64_t((lbo >> 4) & 0x3FFFu) << 16;
    d |= uint64_t((sbo >> 4) & 0x3FFFu) << 32;
    d |= uint64_t(1) << 46;
    d |= uint64_t(2) << 61;
    return d;
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int c0, int c1, int c2,
                                            uint64_t* mbar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];\n" ::
            "r"(tc::smem_u32(dst)),
        "l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(tc::smem_u32(mbar))
        : "memory");
}

__device__ __forceinline__ void commit_to(uint64_t* mbar) { tc::commit(mbar); }

__device__ __forceinline__ void mbar_arrive(uint64_t* mbar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(tc::smem_u32(mbar)) : "memory");
}

__device__ __forceinline__ uint32_t pack2(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}

template <int BN>
__global__ void __launch_bounds__(kThreadsG, 1)
k_gemm_bf16(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b, GemmParams p) {
    constexpr int kStages = Cfg<BN>::kStages;
    constexpr uint32_t kStageBytes = Cfg<BN>::kStageBytes;
    constexpr uint32_t kAccCols = Cfg<BN>::kAccCols;
    constexpr uint32_t kTmemColsG = Cfg<BN>::kTmemCols;
    extern __shared__ __align__(1024) uint8_t smem_g[];
    // the stages start at the first 1024-byte boundary (128-byte swizzle atoms)
    const uint32_t base_s = tc::smem_u32(smem_g);
    uint8_t* stages = smem_g + ((1024u - (base_s & 1023u)) & 1023u);
    uint64_t* full = reinterpret_cast<uint64_t*>(stages + kStages * kStageBytes);
    uint64_t* empty = full + kStages;
    uint64_t* acc_full = empty + kStages;
    uint64_t* acc_empty = acc_full + 2;
    uint64_t* mma_done = acc_empty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
    uint8_t* epi = stages + kStages * kStageBytes + 256;     // epilogue staging (kEpiBytes)

    const int warp = int(threadIdx.x) >> 5, lane = int(threadIdx.x) & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            tc::mbar_init(&full[s], 1);
            tc::mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            tc::mbar_init(&acc_full[a], 1);
            tc::mbar_init(&acc_empty[a], 4);       // one arrival per epilogue warp
        }
        tc::mbar_init(mma_done, 1);
    }
    if (warp == 1) tc::tmem_alloc(tmem_slot, kTmemColsG);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    const int64_t tiles = p.batches * p.tiles_m * p.tiles_n;
    const int kblocks = int((p.K + BK - 1) / BK);

    if (warp == 0) {
        // ---------------- TMA producer
        if (lane == 0) {
            int64_t kc = 0;
            bool ok = true;
            for (int64_t tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x) {
                const int64_t b = tile / (p.tiles_m * p.tiles_n);
                const int64_t rem = tile - b * p.tiles_m * p.tiles_n;
                const int m0 = int((rem / p.tiles_n) * BM), n0 = int((rem % p.tiles_n) * BN);
                for (int kb = 0; kb < kblocks; ++kb, ++kc) {
                    const int s = int(kc % kStages);
                    const uint32_t round = uint32_t(kc / kStages);
                    if (!tc::mbar_wait(&empty[s], (round & 1u) ^ 1u, p.budget_ns)) {
                        ok = false;
                        break;
                    }
                    uint8_t* sa = stages + s * kStageBytes;
                    uint8_t* sb = sa + kATile;
                    tc::mbar_expect_tx(&full[s], kStageBytes);
                    const int k0 = kb * BK;
                    if (p.a_mn_major) {
                        // two 64-row (m) halves of the 128-row tile, each [64 k][64 m]
                        tma_load_3d(sa, &map_a, m0, k0, p.a_batched ? int(b) : 0, &full[s]);
                        tma_load_3d(sa + kATile / 2, &map_a, m0 + 64, k0, p.a_batched ? int(b) : 0, &full[s]);
                    } else {
                        tma_load_3d(sa, &map_a, k0, m0, p.a_batched ? int(b) : 0, &full[s]);
                    }
                    tma_load_3d(sb, &map_b, k0, n0, p.b_batched ? int(b) : 0, &full[s]);
                }
            }
            if (!ok) report_status(p.status, kStatusTimeout);
            // nothing left in flight: the last load of every stage has landed
            for (int64_t j = kc - 1; j >= 0 && j >= kc - kStages; --j)
                tc::mbar_wait(&full[j % kStages], uint32_t(j / kStages) & 1u, p.budget_ns);
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer
        if (lane == 0) {
            const uint32_t idesc = tc::idesc_bf16(BM, BN) | (p.a_mn_major ? (1u << 15) : 0u);
            int64_t kc = 0;
            int it = 0;
            bool ok = true;
            for (int64_t tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x, ++it) {
                const int acc = it & 1;
                const uint32_t use = uint32_t(it >> 1);
                if (!tc::mbar_wait(&acc_empty[acc], (use & 1u) ^ 1u, p.budget_ns)) {
                    ok = false;
                    break;
                }
                tc::fence_after_sync();
                const uint32_t d_tmem = tmem + uint32_t(acc) * kAccCols;
                for (int kb = 0; kb < kblocks; ++kb, ++kc) {
                    const int s = int(kc % kStages);
                    if (!tc::mbar_wait(&full[s], uint32_t(kc / kStages) & 1u, p.budget_ns)) {
                        ok = false;
                        break;
                    }
                    tc::fence_after_sync();
                    const uint32_t sa = tc::smem_u32(stages + s * kStageBytes);
                    const uint32_t sb = sa + kATile;
#pragma unroll
                    for (int ks = 0; ks < BK / 16; ++ks) {
                        // K-major: +32 bytes per 16 elements inside the 128-byte row;
                        // MN-major A: +2 groups of 8 k-rows (1024 bytes each)
                        const uint64_t da = p.a_mn_major ? desc_sw128(sa + uint32_t(ks) * 2048u, kATile / 2, 1024)
                                                         : desc_sw128(sa + uint32_t(ks) * 32u, 16, 1024);
                        const uint64_t db = desc_sw128(sb + uint32_t(ks) * 32u, 16, 1024);
                        tc::mma_bf16(d_tmem, da, db, idesc, (kb > 0 || ks > 0) ? 1u : 0u);
                    }
                    commit_to(&empty[s]);             // the stage is free once these MMAs have read it
                }
                if (!ok) break;
                commit_to(&acc_full[acc]);            // the tile's accumulator is complete
            }
            if (!ok) report_status(p.status, kStatusTimeout);
            // nothing left in flight before tensor memory is released
            commit_to(mma_done);
            if (!tc::mbar_wait(mma_done, 0, p.budget_ns)) report_status(p.status, kStatusTimeout);
        }
    } else {
        // ---------------- epilogue (warps 2..5: lane quarter warp % 4)
        // Accumulator row `row` of the tile is tensor-memory lane `row`.  With
        // 256-wide tiles each thread reads 64 columns of its row, rounds them to
        // bf16 and stages them in shared memory; the warp then stores 4 rows x
        // 128 contiguous bytes per instruction (whole lines instead of 16-byte
        // pieces of 32 rows: half the written sectors).
        const int q = warp & 3;
        const int row = 32 * q + lane;
        uint8_t* sw = epi + (warp - 2) * kEpiWarp;
        int it = 0;
        bool ok = true;
        for (int64_t tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++it) {
            const int acc = it & 1;
            const uint32_t use = uint32_t(it >> 1);
            if (!tc::mbar_wait(&acc_full[acc], use & 1u, p.budget_ns)) {
                ok = false;
                break;
            }
            tc::fence_after_sync();
            const int64_t b = tile / (p.tiles_m * p.tiles_n);
            const int64_t rem = tile - b * p.tiles_m * p.tiles_n;
            const int64_t m_base = (rem / p.tiles_n) * BM + 32 * q;   // this warp's first row
            const int64_t n0 = (rem % p.tiles_n) * BN;
            const int64_t m = m_base + lane;
            const float rb = (p.bias && p.bias_per_row && m < p.M) ? __ldg(p.bias + m) : 0.0f;
            const uint32_t t_acc = tmem + uint32_t(acc) * kAccCols + (uint32_t(32 * q) << 16);
            bf16* cb = p.c + b * p.c_bstride;
            if constexpr (BN == 256) {
#pragma unroll 1
                for (int ch = 0; ch < BN / 64; ++ch) {
                    float v[64];
                    tc::tmem_ld32(t_acc + uint32_t(64 * ch), *reinterpret_cast<float(*)[32]>(v));
                    tc::tmem_ld32(t_acc + uint32_t(64 * ch + 32), *reinterpret_cast<float(*)[32]>(v + 32));
                    tc::tmem_ld_wait();
                    const int64_t n = n0 + 64 * ch;
                    if (p.bias) {
#pragma unroll
                        for (int i = 0; i < 64; ++i)
                            v[i] += p.bias_per_row ? rb : ((n + i < p.N) ? __ldg(p.bias + n + i) : 0.0f);
                    }
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        *reinterpret_cast<uint4*>(sw + lane * kEpiRow + 16 * c) =
                            make_uint4(pack2(v[8 * c], v[8 * c + 1]), pack2(v[8 * c + 2], v[8 * c + 3]),
                                       pack2(v[8 * c + 4], v[8 * c + 5]), pack2(v[8 * c + 6], v[8 * c + 7]));
                    __syncwarp();
                    // round k: rows 4 k + lane / 8, 16-byte chunk lane % 8 of the 64 columns
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const int r = 4 * k + (lane >> 3), c = lane & 7;
                        const uint4 w = *reinterpret_cast<const uint4*>(sw + r * kEpiRow + 16 * c);
                        const int64_t mr = m_base + r, nc = n + 8 * c;
                        if (mr < p.M && nc + 8 <= p.N) *reinterpret_cast<uint4*>(cb + mr * p.ldc + nc) = w;
                    }
                    __syncwarp();
                }
            } else {
                // 128- and 192-wide tiles: each thread stores its row directly (measured faster here)
#pragma unroll 1
                for (int ch = 0; ch < BN / 32; ++ch) {
                    float v[32];
                    tc::tmem_ld32(t_acc + uint32_t(32 * ch), v);
                    tc::tmem_ld_wait();
                    const int64_t n = n0 + 32 * ch;
                    if (m >= p.M || n >= p.N) continue;
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        float bi = rb;
                        if (p.bias && !p.bias_per_row) bi = (n + i < p.N) ? __ldg(p.bias + n + i) : 0.0f;
                        v[i] += bi;
                    }
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        if (n + 8 * g + 8 <= p.N) {
                            const uint4 w = make_uint4(pack2(v[8 * g], v[8 * g + 1]), pack2(v[8 * g + 2], v[8 * g + 3]),
                                                       pack2(v[8 * g + 4], v[8 * g + 5]), pack2(v[8 * g + 6], v[8 * g + 7]));
                            *reinterpret_cast<uint4*>(cb + m * p.ldc + n + 8 * g) = w;
                        }
                    }
                }
            }
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[acc]);
        }
        if (!ok && lane == 0) report_status(p.status, kStatusTimeout);
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 1) tc::tmem_dealloc(tmem, kTmemColsG);
}

// ------------------------------------------------------------------ host
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::mutex g_encode_mutex;

cudaError_t encode_fn(PFN_cuTensorMapEncodeTiled_v12000* out) {
    std::lock_guard<std::mutex> lock(g_encode_mutex);
    if (!g_encode) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
        if (e != cudaSuccess) return e;
        if (q != cudaDriverEntryPointSuccess || !fn) return cudaErrorSymbolNotFound;
        g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    *out = g_encode;
    return cudaSuccess;
}

// 3-D bf16 tensor map, dims (d0 innermost, d1, d2), byte strides of d1 and d2,
// box (b0, b1, 1), 128-byte swizzle; out-of-range elements read as zero.
bool make_map(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t s1, uint64_t s2,
              uint32_t b0, uint32_t b1, std::string* why) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = nullptr;
    cudaError_t e = encode_fn(&enc);
    if (e != cudaSuccess) {
        *why = std::string("cuTensorMapEncodeTiled unavailable: ") + cudaGetErrorString(e);
        return false;
    }
    const cuuint64_t dims[3] = {d0, d1, d2};
    const cuuint64_t strides[2] = {s1, s2};
    const cuuint32_t box[3] = {b0, b1, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        *why = "cuTensorMapEncodeTiled failed (" + std::to_string(int(r)) + ")";
        return false;
    }
    return true;
}

int sm_count() {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms;
}

// Tile width for an M x N output per batch: 256 unless that leaves fewer than
// eight waves of tiles on the SMs (then the last, partly filled wave costs
// more than the narrower tiles do); then 192 where it divides N (fewer
// operand bytes per flop than 128: out_proj at D = 768 64.0 vs 68.1 us), else
// 128.
int pick_bn(int64_t M, int64_t N, int64_t batches) {
    const int64_t tiles256 = batches * ((M + BM - 1) / BM) * ((N + 255) / 256);
    if (tiles256 >= 8 * int64_t(sm_count())) return 256;
    return (N % 192 == 0) ? 192 : 128;
}

template <int BN>
cudaError_t launch_gemm(const CUtensorMap& ma, const CUtensorMap& mb, GemmParams& p, cudaStream_t s) {
    auto kern = k_gemm_bf16<BN>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(Cfg<BN>::kSmem));
    if (e != cudaSuccess) return e;
    const int sms = sm_count();
    p.tiles_m = (p.M + BM - 1) / BM;
    p.tiles_n = (p.N + BN - 1) / BN;
    const int64_t tiles = p.batches * p.tiles_m * p.tiles_n;
    const int64_t grid = tiles < sms ? tiles : sms;
    kern<<<unsigned(grid), kThreadsG, Cfg<BN>::kSmem, s>>>(ma, mb, p);
    return cudaGetLastError();
}

bool al16(const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15u) == 0; }

hyena_status_t check_common(const void* x, const void* W, const float* bias, const void* out, int64_t B, int64_t L,
                            int64_t D) {
    if (!x || !W || !out) return set_last_error_detail(HYENA_ERR_INVALID_ARG, "x, W and out must not be NULL");
    if (B < 1 || L < 1 || D < 1) return set_last_error_detail(HYENA_ERR_INVALID_ARG, "B, L and D must be >= 1");
    if (D % 8 != 0 || L % 8 != 0)
        return set_last_error_detail(HYENA_ERR_UNSUPPORTED_SHAPE, "D and L must be multiples of 8");
    if (B > 65535 || L > (int64_t(1) << 30) || D > 65536)
        return set_last_error_detail(HYENA_ERR_UNSUPPORTED_SHAPE, "B <= 65535, L <= 2^30 and D <= 65536");
    if (!al16(x) || !al16(W) || !al16(out)) return set_last_error_detail(HYENA_ERR_MISALIGNED, "x, W and out must be 16-byte aligned");
    if (bias && (reinterpret_cast<uintptr_t>(bias) & 3u))
        return set_last_error_detail(HYENA_ERR_MISALIGNED, "bias must be 4-byte aligned");
    return HYENA_OK;
}

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
}

}  // namespace
}  // namespace hyena

using namespace hyena;

extern "C" hyena_status_t hyena_in_proj(const void* x, const void* W, const float* bias, void* u, int64_t B,
                                        int64_t L, int64_t D, int order, void* stream) {
    hyena_status_t st = check_common(x, W, bias, u, B, L, D);
    if (st != HYENA_OK) return st;
    if (order < 2 || order > 8) return set_last_error_detail(HYENA_ERR_UNSUPPORTED_SHAPE, "order must be in [2, 8]");
    const int64_t J = int64_t(order + 1) * D;
    if (overlaps(x, size_t(B * L * D) * 2, u, size_t(B * J * L) * 2) || overlaps(W, size_t(J * D) * 2, u, size_t(B * J * L) * 2))
        return set_last_error_detail(HYENA_ERR_INVALID_ARG, "u overlaps x or W");
    std::string why;
    CUtensorMap ma, mb;
    const int bn = pick_bn(J, L, B);
    // A = W_in [J][D] (K-major), B = x [B][L][D] (K-major per position)
    if (!make_map(&ma, W, uint64_t(D), uint64_t(J), 1, uint64_t(D) * 2, uint64_t(J * D) * 2, BK, BM, &why) ||
        !make_map(&mb, x, uint64_t(D), uint64_t(L), uint64_t(B), uint64_t(D) * 2, uint64_t(L * D) * 2, BK, bn, &why))
        return set_last_error_detail(HYENA_ERR_CUDA, why);
    GemmParams p{};
    p.M = J; p.N = L; p.K = D; p.batches = B;
    p.a_mn_major = 0; p.a_batched = 0; p.b_batched = 1;
    p.c = static_cast<bf16*>(u); p.ldc = L; p.c_bstride = J * L;
    p.bias = bias; p.bias_per_row = 1;
    p.budget_ns = kDefaultWaitBudgetNs;
    cudaError_t e = kernel_status_word(&p.status);
    if (e == cudaSuccess)
        e = bn == 256   ? launch_gemm<256>(ma, mb, p, static_cast<cudaStream_t>(stream))
            : bn == 192 ? launch_gemm<192>(ma, mb, p, static_cast<cudaStream_t>(stream))
                        : launch_gemm<128>(ma, mb, p, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return set_last_error_detail(HYENA_ERR_CUDA, std::string("in_proj: ") + cudaGetErrorString(e));
    return set_last_error_detail(HYENA_OK, "");
}

extern "C" hyena_status_t hyena_out_proj(const void* y, const void* W, const float* bias, void* out, int64_t B,
                                         int64_t L, int64_t D, void* stream) {
    hyena_status_t st = check_common(y, W, bias, out, B, L, D);
    if (st != HYENA_OK) return st;
    if (overlaps(y, size_t(B * D * L) * 2, out, size_t(B * L * D) * 2) || overlaps(W, size_t(D * D) * 2, out, size_t(B * L * D) * 2))
        return set_last_error_detail(HYENA_ERR_INVALID_ARG, "out overlaps y or W");
    std::string why;
    CUtensorMap ma, mb;
    const int bn = pick_bn(L, D, B);
    // A = y[b]^T: y [B][D][L] read as [64 l][64 k] boxes (positions contiguous);
    // B = W_out [D][D] (K-major)
    if (!make_map(&ma, y, uint64_t(L), uint64_t(D), uint64_t(B), uint64_t(L) * 2, uint64_t(D * L) * 2, 64, BK, &why) ||
        !make_map(&mb, W, uint64_t(D), uint64_t(D), 1, uint64_t(D) * 2, uint64_t(D * D) * 2, BK, bn, &why))
        return set_last_error_detail(HYENA_ERR_CUDA, why);
    GemmParams p{};
    p.M = L; p.N = D; p.K = D; p.batches = B;
    p.a_mn_major = 1; p.a_batched = 1; p.b_batched = 0;
    p.c = static_cast<bf16*>(out); p.ldc = D; p.c_bstride = L * D;
    p.bias = bias; p.bias_per_row = 0;
    p.budget_ns = kDefaultWaitBudgetNs;
    cudaError_t e = kernel_status_word(&p.status);
    if (e == cudaSuccess)
        e = bn == 256   ? launch_gemm<256>(ma, mb, p, static_cast<cudaStream_t>(stream))
            : bn == 192 ? launch_gemm<192>(ma, mb, p, static_cast<cudaStream_t>(stream))
                        : launch_gemm<128>(ma, mb, p, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return set_last_error_detail(HYENA_ERR_CUDA, std::string("out_proj: ") + cudaGetErrorString(e));
    return set_last_error_detail(HYENA_OK, "");
}
