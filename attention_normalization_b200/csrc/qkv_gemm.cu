// QKV projection GEMM with Phase A partial squared sums in the epilogue
// (tcgen05 + TMA + TMEM, sm_100a).  The kernel's structure is described in
// qkv_gemm.cuh.

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "qkv_gemm.cuh"

namespace qkn {
namespace gemm {
namespace {

// Set by a wait that ran out; read and cleared by read_and_clear_timeout.
__device__ int g_timeout_code = 0;

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ---------------------------------------------------------------- mbarriers
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(bar), "r"(parity)
        : "memory");
    return done != 0;
}

// True once the phase of parity `parity` has completed; false when
// `timeout_ns` of global time passed first.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, uint64_t timeout_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    for (;;) {
        for (int i = 0; i < 32; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (global_ns() - t0 > timeout_ns) return false;
    }
}

// ---------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int32_t c0, int32_t c1,
                                            uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
        "[%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar)
        : "memory");
}

// With a CTA pair the load lands in this CTA's shared memory and its bytes are
// counted on `bar`, the leader CTA's barrier (a shared::cluster address).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap *map, int32_t c0, int32_t c1,
                                                 uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, "
        "%3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar)
        : "memory");
}

// ---------------------------------------------------------------- clusters
__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// The shared::cluster address of the variable at shared::cta address `addr`
// in the cluster's CTA `rank`.
__device__ __forceinline__ uint32_t map_to_cta(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}

// All threads of both CTAs of the pair.
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

__device__ __forceinline__ void prefetch_map(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---------------------------------------------------------------- tcgen05
__device__ __forceinline__ void fence_before_sync() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_after_sync() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptor of a K-major operand tile stored as rows of
// 128 bytes with the 128-byte swizzle (what a TMA box of 64 bf16 x rows with
// CU_TENSOR_MAP_SWIZZLE_128B writes): start address >> 4 in bits 0-13,
// leading-dimension offset 1 (unused by swizzled K-major layouts), stride
// between 8-row groups 1024 bytes (>> 4 in bits 32-45), descriptor version 1
// (bits 46-47), base offset 0 (atoms are 1024-byte aligned), layout type 2 =
// 128-byte swizzle (bits 61-63).
__device__ __forceinline__ uint64_t sw128_kmajor_desc(uint32_t saddr) {
    return static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4) | (static_cast<uint64_t>(1) << 16) |
           (static_cast<uint64_t>(1024 >> 4) << 32) | (static_cast<uint64_t>(1) << 46) |
           (static_cast<uint64_t>(2) << 61);
}

// Instruction descriptor of tcgen05.mma kind::f16: fp32 accumulator (bits
// 4-5 = 1), A and B bf16 (bits 7-9 and 10-12 = 1), both K-major (bits 15, 16
// = 0), N >> 3 in bits 17-22, M >> 4 in bits 24-28.
constexpr uint32_t kIdescBf16 = (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(kBN >> 3) << 17) |
                                (static_cast<uint32_t>((kBM * kCta) >> 4) << 24);

__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::%5.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "n"(kCta)
        : "memory");
}

// The mbarrier receives one arrival when every tcgen05.mma this thread issued
// so far has completed; with a CTA pair, the barrier at the same offset in
// both CTAs does.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
    if constexpr (kCta == 1) {
        asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                     : "memory");
    } else {
        asm volatile(
            "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
                bar),
            "h"(static_cast<uint16_t>(0x3))
            : "memory");
    }
}

// 32 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]),
          "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]),
          "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void record_timeout(int code, int *flag) {
    atomicExch(&g_timeout_code, code);
    *flag = 1;
}

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Barrier among the epilogue warps only (named barrier 1; 0 is __syncthreads).
__device__ __forceinline__ void epilogue_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(kEpiWarps * 32) : "memory");
}

// True on every epilogue thread iff `ok` holds on all of them (a named
// barrier with an AND reduction), so all epilogue warps take the same branch.
__device__ __forceinline__ bool epilogue_all(bool ok) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, 1, %2, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(static_cast<uint32_t>(ok)), "n"(kEpiWarps * 32)
        : "memory");
    return r != 0;
}

// This CTA's j-th tile: work unit u = cluster + j * clusters (a unit is one
// MMA's 128 * kCta tokens x 256 columns); the CTA takes token tile
// m_unit * kCta + rank of it.  Units are rastered in groups of group_units
// token blocks: within a group the token block runs fastest, then the column
// tile, then the group (the last group may hold fewer token blocks).  One
// group spanning all token blocks lets the units running at one time share a
// few W tiles while X stays in L2; smaller groups keep a wave's X blocks and
// W tiles in L2 together when neither operand fits on its own.
struct TileRef {
    int m_tile, n_tile;
};
__host__ __device__ __forceinline__ void unit_tile(const GemmParams &p, int u, int *m_unit, int *n_tile) {
    const int span = p.group_units * p.n_tiles;
    const int g = u / span;
    const int v = u - g * span;
    const int first = g * p.group_units;
    const int rows = p.group_units < p.m_units - first ? p.group_units : p.m_units - first;
    *m_unit = first + v % rows;
    *n_tile = v / rows;
}
__device__ __forceinline__ TileRef cta_tile(const GemmParams &p, int j, int rank) {
    const int clusters = static_cast<int>(gridDim.x) / kCta;
    int m_unit, n_tile;
    unit_tile(p, static_cast<int>(blockIdx.x) / kCta + j * clusters, &m_unit, &n_tile);
    return TileRef{m_unit * kCta + rank, n_tile};
}
__device__ __forceinline__ int cta_tile_count(const GemmParams &p) {
    const int clusters = static_cast<int>(gridDim.x) / kCta;
    const int c = static_cast<int>(blockIdx.x) / kCta;
    return c < p.num_units ? (p.num_units - c + clusters - 1) / clusters : 0;
}

}  // namespace

__global__ void __launch_bounds__(kThreads, 1)
    qkv_gemm_stats_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                          const __grid_constant__ GemmParams p) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ int s_abort;      // a wait in this CTA ran out
    __shared__ int s_consumed;   // k-blocks (over all tiles) whose MMAs were issued
    __shared__ int s_issued;     // k-blocks (over all tiles) whose TMA loads were issued
    __shared__ float s_half[2][kBM];  // second-half squared sums, by tile parity

    // 1024-byte aligned ring: A stages, then B stages, then the mbarriers:
    // full[kStages], empty[kStages], acc_full[2], acc_empty[2].  The layout
    // is the same in both CTAs of a pair, so one offset names a barrier in
    // either.
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    const uint32_t a_base = base;
    const uint32_t b_base = base + kStages * kABytes;
    const uint32_t bars = base + kStages * kStageBytes;
    auto full_bar = [&](int s) { return bars + 8u * s; };
    auto empty_bar = [&](int s) { return bars + 8u * (kStages + s); };
    auto acc_full_bar = [&](int b) { return bars + 8u * (2 * kStages + b); };
    auto acc_empty_bar = [&](int b) { return bars + 8u * (2 * kStages + 2 + b); };
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem_raw + (bars - raw) + 8 * (2 * kStages + 4));

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int rank = kCta == 2 ? static_cast<int>(cluster_rank()) : 0;
    const bool leader = rank == 0;  // issues the MMAs and owns the barriers they wait on
    const int n_tiles_cta = cta_tile_count(p);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(full_bar(s), 1);   // the leader's expect-tx arrival; bytes of both CTAs
            mbar_init(empty_bar(s), 1);  // one tcgen05.commit
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(acc_full_bar(b), 1);                   // one tcgen05.commit per tile
            mbar_init(acc_empty_bar(b), kEpiWarps * kCta);   // every epilogue warp of the group
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        prefetch_map(&tmap_x);
        prefetch_map(&tmap_w);
        s_abort = 0;
        s_consumed = 0;
        s_issued = 0;
    }
    if (warp == 1) {  // both CTAs of a pair allocate, with the same warp and address
        if constexpr (kCta == 1) {
            asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                             smem_u32(tmem_slot)),
                         "r"(kTmemCols)
                         : "memory");
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
        } else {
            asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                             smem_u32(tmem_slot)),
                         "r"(kTmemCols)
                         : "memory");
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
        }
    }
    fence_before_sync();
    __syncthreads();
    if constexpr (kCta == 2) cluster_sync();  // the peer's barriers are initialized before any remote use
    fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    pdl_wait();  // X may come from the previous kernel in the stream; qkv may still be read by it

    if (warp == 0) {
        if (lane == 0) {  // ---------------------------------------------- TMA producer (each CTA)
            int it = 0;   // k-blocks issued so far, over all of this CTA's tiles
            for (int j = 0; j < n_tiles_cta; ++j) {
                const TileRef tr = cta_tile(p, j, rank);
                for (int kb = 0; kb < p.k_blocks; ++kb, ++it) {
                    const int s = it % kStages;
                    const int round = it / kStages;
                    if (round > 0 && !mbar_wait(empty_bar(s), (round - 1) & 1, p.timeout_ns)) {
                        record_timeout(kErrProducer, &s_abort);
                        break;
                    }
                    if (leader) mbar_expect_tx(full_bar(s), kTxBytes);
                    const int ax = kb * kBK, ay = tr.m_tile * kBM;
                    const int by = tr.n_tile * kBN + rank * kBNLocal;
                    if constexpr (kCta == 1) {
                        tma_load_2d(a_base + s * kABytes, &tmap_x, ax, ay, full_bar(s));
                        tma_load_2d(b_base + s * kBBytes, &tmap_w, ax, by, full_bar(s));
                    } else {
                        const uint32_t lbar = map_to_cta(full_bar(s), 0);
                        tma_load_2d_pair(a_base + s * kABytes, &tmap_x, ax, ay, lbar);
                        tma_load_2d_pair(b_base + s * kBBytes, &tmap_w, ax, by, lbar);
                    }
                }
            }
            s_issued = it;
        }
    } else if (warp == 1) {
        if (leader && lane == 0) {  // ------------------------------------ MMA issuer (leader CTA)
            int it = 0;   // k-blocks consumed so far
            bool ok = true;
            for (int j = 0; ok && j < n_tiles_cta; ++j) {
                const int b = j & 1;
                const int use = j >> 1;  // earlier uses of accumulator b
                if (use > 0 && !mbar_wait(acc_empty_bar(b), (use - 1) & 1, p.timeout_ns)) {
                    record_timeout(kErrMma, &s_abort);
                    break;
                }
                fence_after_sync();
                const uint32_t acc = tmem + static_cast<uint32_t>(b * kAccCols);
                for (int kb = 0; kb < p.k_blocks; ++kb, ++it) {
                    const int s = it % kStages;
                    if (!mbar_wait(full_bar(s), (it / kStages) & 1, p.timeout_ns)) {
                        record_timeout(kErrMma, &s_abort);
                        ok = false;
                        break;
                    }
                    fence_after_sync();
                    const uint32_t a_s = a_base + s * kABytes;
                    const uint32_t b_s = b_base + s * kBBytes;
#pragma unroll
                    for (int k = 0; k < kBK / kUmmaK; ++k)
                        umma_bf16(acc, sw128_kmajor_desc(a_s + k * kUmmaK * 2),
                                  sw128_kmajor_desc(b_s + k * kUmmaK * 2), kIdescBf16, (kb | k) != 0 ? 1u : 0u);
                    umma_commit(empty_bar(s));
                }
                umma_commit(acc_full_bar(b));  // also after a timeout, so the epilogues are not left waiting
            }
            s_consumed = it;
        }
        __syncwarp();
    } else {  // ------------------------------------------------------------ epilogue (each CTA)
        const int quarter = warp & 3;          // TMEM lanes this warp may read
        const int half = (warp - 2) >> 2;      // which column range of the tile (0 with 4 warps)
        const int rl = quarter * 32 + lane;    // row within the tile
        // the leader's acc_empty barriers: every epilogue warp of the group arrives there
        const uint32_t acc_empty_leader[2] = {kCta == 2 ? map_to_cta(acc_empty_bar(0), 0) : acc_empty_bar(0),
                                              kCta == 2 ? map_to_cta(acc_empty_bar(1), 0) : acc_empty_bar(1)};
        for (int j = 0; j < n_tiles_cta; ++j) {
            const int b = j & 1;
            const int use = j >> 1;
            bool ok = mbar_wait(acc_full_bar(b), use & 1, p.timeout_ns);
            if (!ok) record_timeout(kErrEpilogue, &s_abort);
            // the same decision in every epilogue warp, so the named barriers below always match
            if (!epilogue_all(ok && p.k_blocks > 0)) break;
            fence_after_sync();
            const TileRef tr = cta_tile(p, j, rank);
            const int m_tile = tr.m_tile, n_tile = tr.n_tile;
            const bool tile_live = m_tile < p.m_tiles;  // the pair's second token tile may lie past T
            const int64_t row = static_cast<int64_t>(m_tile) * kBM + rl;
            const bool live = row < p.T;
            const int col0 = half * kEpiCols;
            char *orow = p.qkv + (live ? row : 0) * p.qkv_stride_bytes + (static_cast<int64_t>(n_tile) * kBN + col0) * 2;
            const uint32_t taddr = tmem + (static_cast<uint32_t>(quarter * 32) << 16) +
                                   static_cast<uint32_t>(b * kAccCols + col0);
            float ss = 0.0f;
#pragma unroll 1
            for (int c = 0; c < kEpiCols / 32; ++c) {
                uint32_t r[32];
                tmem_ld32(taddr + c * 32, r);
                uint32_t packed[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const __nv_bfloat162 h =
                        __float22bfloat162_rn(make_float2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1])));
                    const float lo = __low2float(h), hi = __high2float(h);
                    ss = fmaf(lo, lo, ss);
                    ss = fmaf(hi, hi, ss);
                    packed[i] = *reinterpret_cast<const uint32_t *>(&h);
                }
                if (live) {
                    uint4 *dst = reinterpret_cast<uint4 *>(orow + c * 64);
#pragma unroll
                    for (int v = 0; v < 4; ++v)
                        dst[v] = make_uint4(packed[4 * v], packed[4 * v + 1], packed[4 * v + 2], packed[4 * v + 3]);
                }
            }
            // The accumulator has been read: hand it back to the MMA thread.
            fence_before_sync();
            __syncwarp();
            if (lane == 0) {
                if constexpr (kCta == 1)
                    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(acc_empty_bar(b)) : "memory");
                else
                    mbar_arrive_cluster(acc_empty_leader[b]);
            }

            const int tensor = n_tile < p.q_tiles ? 0 : (n_tile < p.q_tiles + p.k_tiles ? 1 : -1);
            if (tensor >= 0 && tile_live) {  // Q or K tile: its partial sums (V columns have none)
                if (kEpiSplit == 2 && half == 1) s_half[b][rl] = ss;
                if (kEpiSplit == 2) epilogue_sync();
                if (half == 0 && live) {
                    const float total = kEpiSplit == 2 ? ss + s_half[b][rl] : ss;
                    if (tensor == 0) {
                        if (p.q_sumsq) p.q_sumsq[static_cast<int64_t>(n_tile) * p.T + row] = total;
                    } else {
                        if (p.k_sumsq) p.k_sumsq[static_cast<int64_t>(n_tile - p.q_tiles) * p.T + row] = total;
                    }
                }
                epilogue_sync();  // s_half[b] has been read before the tile after next reuses it
            }
        }
    }

    fence_before_sync();
    __syncthreads();
    if (threadIdx.x == 0 && s_abort && leader) {
        // After a timeout, loads the MMA thread never consumed may still be in
        // flight (both CTAs' bytes count on the leader's barriers): let them
        // land, bounded, before shared memory is released.
        for (int it = s_consumed; it < s_issued; ++it)
            (void)mbar_wait(full_bar(it % kStages), (it / kStages) & 1, p.timeout_ns);
    }
    if constexpr (kCta == 2) cluster_sync();  // no CTA leaves while its peer may still use its memory
    if (warp == 1) {
        fence_after_sync();
        if constexpr (kCta == 1)
            asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                         : "memory");
        else
            asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                         : "memory");
    }
}

// ------------------------------------------------------------------ host side
namespace {

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;
cudaError_t g_encode_status = cudaSuccess;

cudaError_t encoder(PFN_cuTensorMapEncodeTiled_v12000 *fn) {
    std::call_once(g_encode_once, [] {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        g_encode_status = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q);
        if (g_encode_status == cudaSuccess && (q != cudaDriverEntryPointSuccess || !f))
            g_encode_status = cudaErrorSymbolNotFound;
        g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    });
    *fn = g_encode;
    return g_encode_status;
}

// A row-major bf16 matrix [outer][inner] with rows `stride_elems` apart, read
// in boxes of box_outer rows x 64 columns with the 128-byte swizzle; reads
// beyond the matrix return zeros.
bool encode_bf16_rows(PFN_cuTensorMapEncodeTiled_v12000 fn, CUtensorMap *map, const void *base, int64_t inner,
                      int64_t outer, int64_t stride_elems, uint32_t box_outer) {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(outer)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(stride_elems) * 2};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(kBK), box_outer};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

constexpr int kMaxDevices = 64;
bool g_smem_set[kMaxDevices] = {};
int g_groups[kMaxDevices] = {};  // resident CTA groups per device
std::mutex g_smem_mu;

// Token blocks per raster group (1 .. m_units) for `clusters` CTA groups
// running at once, by what must stay in L2 (half of it, leaving room for the
// stored tiles):
//   * X fits: one group -- the token blocks run fastest, X stays resident and
//     each W tile is read by the units of about one wave;
//   * else W fits: one token block per group -- each X block is read once by
//     the units that need it, one after another, and W stays resident;
//   * else the G that makes a wave's distinct X blocks + W tiles, G +
//     ceil(clusters / G), smallest (about sqrt(clusters)), so a wave's
//     operands fit in L2 together.
// (One B200, projection + QK-Norm, D = 4096: at T = 16384 this order took
// 597 us against 731 us for one group with Hq = 4096, Hk = Hv = 1024, and
// 1235 us against 1391 us with Hq = Hk = Hv = 4096; at T = 4096 one group was
// best or equal.)
int raster_group_units(int m_units, int D, int N, int clusters, int l2_bytes) {
    int g = m_units;
    if (kGroupM >= 0) {
        g = kGroupM == 0 ? m_units : kGroupM;
    } else {
        const double budget = 0.5 * static_cast<double>(l2_bytes > 0 ? l2_bytes : (64 << 20));
        const double x_bytes = static_cast<double>(m_units) * kBM * kCta * D * 2.0;
        const double w_bytes = static_cast<double>(N) * D * 2.0;
        if (x_bytes <= budget) {
            g = m_units;
        } else if (w_bytes <= budget) {
            g = 1;
        } else {
            int best = 1, best_cost = 1 + clusters;
            for (int c = 2; c <= m_units && c <= clusters; ++c) {
                const int cost = c + (clusters + c - 1) / c;
                if (cost < best_cost) best = c, best_cost = cost;
            }
            g = best;
        }
    }
    return g < 1 ? 1 : (g > m_units ? m_units : g);
}

// The launch configuration shared by the launch and the occupancy query.
void base_config(cudaLaunchConfig_t *cfg, cudaLaunchAttribute (&attr)[2], cudaStream_t stream) {
    *cfg = cudaLaunchConfig_t{};
    cfg->blockDim = dim3(kThreads);
    cfg->dynamicSmemBytes = kSmemBytes;
    cfg->stream = stream;
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = kCta;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg->attrs = attr;
    cfg->numAttrs = kCta == 2 ? 2 : 1;
}

}  // namespace

void schedule_qkv_gemm(GemmParams *p, int32_t D, int32_t N, int clusters, int64_t l2_bytes) {
    const int units = p->num_units < clusters ? p->num_units : clusters;
    p->group_units = raster_group_units(p->m_units, D, N, units > 0 ? units : 1,
                                        static_cast<int>(l2_bytes > (int64_t(1) << 30) ? (int64_t(1) << 30) : l2_bytes));
}

cudaError_t qkv_gemm_clusters(int *clusters, const char **what) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        *what = "cudaGetDevice";
        return e;
    }
    {
        std::lock_guard<std::mutex> lk(g_smem_mu);
        if (dev < 0 || dev >= kMaxDevices || !g_smem_set[dev]) {
            e = cudaFuncSetAttribute(qkv_gemm_stats_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
            if (e != cudaSuccess) {
                *what = "cudaFuncSetAttribute(max dynamic shared memory)";
                return e;
            }
            if (dev >= 0 && dev < kMaxDevices) g_smem_set[dev] = true;
        }
    }
    // Persistent: one CTA per SM (its shared memory allows no second one), as
    // many CTA groups as can be resident at once, so every group runs from
    // the start (a group that waited for a free SM would finish last).
    cudaLaunchConfig_t cfg;
    cudaLaunchAttribute attr[2];
    base_config(&cfg, attr, nullptr);
    int groups = 0;
    {
        std::lock_guard<std::mutex> lk(g_smem_mu);
        if (dev >= 0 && dev < kMaxDevices && g_groups[dev] > 0) groups = g_groups[dev];
    }
    if (groups == 0) {
        if constexpr (kCta == 1) {
            e = cudaDeviceGetAttribute(&groups, cudaDevAttrMultiProcessorCount, dev);
            if (e != cudaSuccess) {
                *what = "cudaDeviceGetAttribute(multiprocessor count)";
                return e;
            }
        } else {
            cfg.gridDim = dim3(kCta);
            e = cudaOccupancyMaxActiveClusters(&groups, reinterpret_cast<const void *>(qkv_gemm_stats_kernel), &cfg);
            if (e != cudaSuccess) {
                *what = "cudaOccupancyMaxActiveClusters";
                return e;
            }
        }
        if (groups < 1) {
            *what = "no resident CTA group";
            return cudaErrorInvalidConfiguration;
        }
        std::lock_guard<std::mutex> lk(g_smem_mu);
        if (dev >= 0 && dev < kMaxDevices) g_groups[dev] = groups;
    }
    *clusters = groups;
    return cudaSuccess;
}

cudaError_t launch_qkv_gemm(const void *x, int64_t x_stride, const void *w, int64_t w_stride, int32_t D,
                            int32_t N, const GemmParams &p, cudaStream_t stream, const char **what) {
    PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    cudaError_t e = encoder(&fn);
    if (e != cudaSuccess) {
        *what = "cuTensorMapEncodeTiled entry point";
        return e;
    }
    CUtensorMap tx, tw;
    if (!encode_bf16_rows(fn, &tx, x, D, p.T, x_stride, kBM) ||
        !encode_bf16_rows(fn, &tw, w, D, N, w_stride, kBNLocal)) {  // each CTA stages kBNLocal W rows
        *what = "cuTensorMapEncodeTiled";
        return cudaErrorInvalidValue;
    }
    int groups = 0;
    if ((e = qkv_gemm_clusters(&groups, what)) != cudaSuccess) return e;
    int dev = 0, l2 = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) {
        *what = "cudaGetDevice";
        return e;
    }
    if ((e = cudaDeviceGetAttribute(&l2, cudaDevAttrL2CacheSize, dev)) != cudaSuccess) {
        *what = "cudaDeviceGetAttribute(L2 cache size)";
        return e;
    }
    cudaLaunchConfig_t cfg;
    cudaLaunchAttribute attr[2];
    base_config(&cfg, attr, stream);
    const int units = p.num_units < groups ? p.num_units : groups;
    cfg.gridDim = dim3(static_cast<unsigned>((units > 0 ? units : 1) * kCta));
    GemmParams q = p;
    schedule_qkv_gemm(&q, D, N, groups, l2);
    void *args[] = {&tx, &tw, &q};
    e = cudaLaunchKernelExC(&cfg, reinterpret_cast<const void *>(qkv_gemm_stats_kernel), args);
    if (e != cudaSuccess) *what = "cudaLaunchKernelExC";
    return e;
}

cudaError_t read_and_clear_timeout(int *code) {
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return e;
    int v = 0;
    if ((e = cudaMemcpyFromSymbol(&v, g_timeout_code, sizeof(int))) != cudaSuccess) return e;
    const int zero = 0;
    if ((e = cudaMemcpyToSymbol(g_timeout_code, &zero, sizeof(int))) != cudaSuccess) return e;
    *code = v;
    return cudaSuccess;
}

}  // namespace gemm
}  // namespace qkn
