// ep_gemm.cuh -- the experts between dispatch and combine: grouped matrix
// multiplications on the fifth-generation tensor cores.
//
// "[feat] A5 deep fused moe supported" runs grouped matrix multiplications of
// the experts between its dispatch and its combine.  Here each expert e is one
// linear map W_e [N][H]: for the rows r of expert e in the packed receive
// layout (expert_offset[e] .. + count[e]),
//   y[r, :] = bf16_rne( x[r, :] . W_e^T ),  fp32 accumulation.
// Three kernels: expert_gemm_kernel (bf16, below), expert_gemm2_kernel (bf16
// on CTA pairs with the two-CTA MMA) and expert_gemm_mx_kernel (MXFP8 / MXFP4
// codes with e8m0 block scales, the block-scaled MMA), each described where
// it is defined.
//
// bf16: tiles of 128 rows x 256 columns, 64-element K steps.  A persistent grid
// (one block per SM) walks the tiles of all experts; in each block
//   warp 0        loads A and B K-steps with TMA (128-byte swizzle) into a
//                 ring of kGemmStages shared-memory stages;
//   warp 1        allocates 2 x 256 TMEM columns (two fp32 accumulators: all
//                 of the SM's TMEM) and one lane issues tcgen05.mma
//                 (cta_group::1, kind::f16, M=128, N=256, K=16 per
//                 instruction), committing each stage back to
//                 the loader and each finished accumulator to the epilogue;
//   warps 2 - 5   read the accumulator rows (tcgen05.ld, one TMEM lane
//                 quarter per warp), round to bf16 and store the tile's valid
//                 rows, then hand the accumulator back.
// Every wait on an mbarrier gives up after 2 s of %globaltimer: the block then
// records kDevTimeout in the status word, drains its copies and MMAs in
// flight (with the same bound), frees its TMEM and returns.
#pragma once

#include <cuda.h>

#include "ep_device.cuh"
#include "ep_mbar.cuh"

namespace ep {

constexpr int kGemmBM = 128, kGemmBN = 256, kGemmBK = 64, kGemmStages = 4;
constexpr int kGemmThreads = 192;
constexpr int kGemmTileBytesA = kGemmBM * kGemmBK * 2;  // 16 KB
constexpr int kGemmTileBytesB = kGemmBN * kGemmBK * 2;  // 32 KB
constexpr int kGemmMaxExperts = 1024;

struct GemmArgs {
    int E, H, N;
    int ntn;                 // N / kGemmBN
    const int64_t *eo;       // [E+1] first row of each expert (packed layout)
    const int64_t *cnt;      // [E] rows of each expert
    uint16_t *y;             // [rows][N] bf16
    uint32_t *status;
};

// dynamic shared memory: stages (1024-byte aligned for the swizzle), then the
// barriers, the TMEM base, an abort flag and the per-expert tile prefix
__host__ __device__ constexpr size_t gemm_smem_bytes() {
    return 1024 + (size_t)kGemmStages * (kGemmTileBytesA + kGemmTileBytesB) +
           (2 * kGemmStages + 5) * 8 + 16 + (kGemmMaxExperts + 1) * 4 + 256;
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int c0, int c1,
                                            uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar)
        : "memory");
}
// shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart (leading offset 1, stride offset 64 in 16-byte units,
// descriptor version 1, layout type 2)
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t saddr) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)64 << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
// instruction descriptor: fp32 accumulator, bf16 A and B, both K-major, N, M
__host__ __device__ constexpr uint32_t umma_idesc_bf16(int M, int N) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}
__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void umma_commit(uint32_t bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
        : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15}, [%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
          "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]),
          "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(taddr));
    // the registers are operands of the wait, so no use moves above it
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(v[0]), "+r"(v[1]), "+r"(v[2]), "+r"(v[3]), "+r"(v[4]), "+r"(v[5]),
                   "+r"(v[6]), "+r"(v[7]), "+r"(v[8]), "+r"(v[9]), "+r"(v[10]), "+r"(v[11]),
                   "+r"(v[12]), "+r"(v[13]), "+r"(v[14]), "+r"(v[15])
                 :
                 : "memory");
}

// 32 consecutive fp32 columns of this warp's 32 TMEM lanes, one wait
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
        "%28, %29, %30, %31}, [%32];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
          "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]),
          "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]),
          "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]),
          "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]),
          "=r"(v[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(v[0]), "+r"(v[1]), "+r"(v[2]), "+r"(v[3]), "+r"(v[4]), "+r"(v[5]),
                   "+r"(v[6]), "+r"(v[7]), "+r"(v[8]), "+r"(v[9]), "+r"(v[10]), "+r"(v[11]),
                   "+r"(v[12]), "+r"(v[13]), "+r"(v[14]), "+r"(v[15]), "+r"(v[16]), "+r"(v[17]),
                   "+r"(v[18]), "+r"(v[19]), "+r"(v[20]), "+r"(v[21]), "+r"(v[22]), "+r"(v[23]),
                   "+r"(v[24]), "+r"(v[25]), "+r"(v[26]), "+r"(v[27]), "+r"(v[28]), "+r"(v[29]),
                   "+r"(v[30]), "+r"(v[31])
                 :
                 : "memory");
}

// 16 fp32 accumulator columns of one row -> 16 bf16 (round to nearest even)
__device__ __forceinline__ void store_bf16x16(uint16_t *dst, const uint32_t (&v)[16]) {
    uint4 lo, hi;
    lo.x = pack_bf16x2(__uint_as_float(v[0]), __uint_as_float(v[1]));
    lo.y = pack_bf16x2(__uint_as_float(v[2]), __uint_as_float(v[3]));
    lo.z = pack_bf16x2(__uint_as_float(v[4]), __uint_as_float(v[5]));
    lo.w = pack_bf16x2(__uint_as_float(v[6]), __uint_as_float(v[7]));
    hi.x = pack_bf16x2(__uint_as_float(v[8]), __uint_as_float(v[9]));
    hi.y = pack_bf16x2(__uint_as_float(v[10]), __uint_as_float(v[11]));
    hi.z = pack_bf16x2(__uint_as_float(v[12]), __uint_as_float(v[13]));
    hi.w = pack_bf16x2(__uint_as_float(v[14]), __uint_as_float(v[15]));
    st_v4(dst, lo);
    st_v4(dst + 8, hi);
}

// tile t of the walk -> expert, first row and first column (t < prefix[E]).
// Within an expert the row tiles vary fastest: the blocks that read the same
// weight columns run side by side, so those columns come from DRAM once.
__device__ __forceinline__ void gemm_tile(const int *prefix, int E, int ntn, int t, int &e,
                                          int &m0, int &n0, int bn = kGemmBN, int bm = kGemmBM) {
    int lo = 0, hi = E - 1;  // the last e with prefix[e] <= t
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (prefix[mid] <= t) lo = mid;
        else hi = mid - 1;
    }
    e = lo;
    const int local = t - prefix[e];
    const int mt = (prefix[e + 1] - prefix[e]) / ntn;  // row tiles of expert e
    m0 = (local % mt) * bm;
    n0 = (local / mt) * bn;
}

// tiles per expert, exclusive prefix into prefix[0..E] (one warp; each lane
// takes a run of experts)
__device__ __forceinline__ void tile_prefix(int *prefix, int E, const int64_t *cnt, int ntn,
                                            int lane, int bm = kGemmBM) {
    const int per = (E + 31) / 32;
    int sum = 0;
    for (int i = 0; i < per; i++) {
        const int e = lane * per + i;
        if (e < E) sum += (int)((cnt[e] + bm - 1) / bm) * ntn;
    }
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(kFull, incl, o);
        if (lane >= o) incl += v;
    }
    int run = incl - sum;
    for (int i = 0; i < per; i++) {
        const int e = lane * per + i;
        if (e < E) {
            prefix[e] = run;
            run += (int)((cnt[e] + bm - 1) / bm) * ntn;
        }
    }
    if (lane == 31) prefix[E] = incl;
}

__global__ void __launch_bounds__(kGemmThreads, 1)
    expert_gemm_kernel(const __grid_constant__ CUtensorMap tm_a,
                       const __grid_constant__ CUtensorMap tm_b, GemmArgs a) {
    extern __shared__ uint8_t gsm_raw[];
    uint8_t *gsm = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(gsm_raw) + 1023) & ~(uintptr_t)1023);
    uint8_t *sA = gsm;
    uint8_t *sB = gsm + kGemmStages * kGemmTileBytesA;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sB + kGemmStages * kGemmTileBytesB);
    uint64_t *full = bars, *empty = bars + kGemmStages;
    uint64_t *accfull = bars + 2 * kGemmStages, *accempty = accfull + 2;
    uint64_t *drain = accempty + 2;
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(drain + 1);
    volatile uint32_t *s_abort = s_tmem + 1;
    int *prefix = reinterpret_cast<int *>(s_tmem + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int E = a.E;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kGemmStages; s++) {
            mbar_init(smem_addr(&full[s]), 1);
            mbar_init(smem_addr(&empty[s]), 1);
        }
        for (int b = 0; b < 2; b++) {
            mbar_init(smem_addr(&accfull[b]), 1);
            mbar_init(smem_addr(&accempty[b]), 128);
        }
        mbar_init(smem_addr(drain), 1);
        *s_abort = 0u;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {  // the whole warp: 2 x kGemmBN columns
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_addr(s_tmem)),
                     "r"(2 * kGemmBN));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    pdl_enter();
    if (warp == 0) tile_prefix(prefix, E, a.cnt, a.ntn, lane);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *s_tmem;
    const int total = prefix[E];
    const int kblocks = a.H / kGemmBK;

    if (warp == 0 && lane == 0) {
        // ---- loader
        int it = 0;
        for (int t = blockIdx.x; t < total && !*s_abort; t += gridDim.x) {
            int e, m0, n0;
            gemm_tile(prefix, E, a.ntn, t, e, m0, n0);
            const int arow = (int)a.eo[e] + m0, brow = e * a.N + n0;
            for (int kb = 0; kb < kblocks; kb++, it++) {
                const int s = it % kGemmStages, r = it / kGemmStages;
                if (!mbar_wait(smem_addr(&empty[s]), (r & 1) ^ 1)) {
                    *s_abort = 1u;
                    atomicOr(a.status, kDevTimeout);
                    break;
                }
                const uint32_t fb = smem_addr(&full[s]);
                mbar_expect_tx(fb, kGemmTileBytesA + kGemmTileBytesB);
                tma_load_2d(smem_addr(sA + s * kGemmTileBytesA), &tm_a, kb * kGemmBK, arow, fb);
                tma_load_2d(smem_addr(sB + s * kGemmTileBytesB), &tm_b, kb * kGemmBK, brow, fb);
            }
        }
        // copies still in flight land before the block can leave: wait for the
        // last fill of every stage that was filled (bounded)
        for (int j = 0; j < kGemmStages && j < it; j++) {
            const int i2 = it - 1 - j, s = i2 % kGemmStages, r = i2 / kGemmStages;
            if (!mbar_wait(smem_addr(&full[s]), r & 1)) atomicOr(a.status, kDevTimeout);
        }
    } else if (warp == 1 && lane == 0) {
        // ---- MMA issue
        const uint32_t idesc = umma_idesc_bf16(kGemmBM, kGemmBN);
        int it = 0, tc = 0;
        for (int t = blockIdx.x; t < total && !*s_abort; t += gridDim.x, tc++) {
            const int acc = tc & 1, use = tc >> 1;
            if (!mbar_wait(smem_addr(&accempty[acc]), (use & 1) ^ 1)) {
                *s_abort = 1u;
                atomicOr(a.status, kDevTimeout);
                break;
            }
            tc_fence_after();
            const uint32_t d = tmem_base + (uint32_t)(acc * kGemmBN);
            bool ok = true;
            for (int kb = 0; kb < kblocks; kb++, it++) {
                const int s = it % kGemmStages, r = it / kGemmStages;
                if (!mbar_wait(smem_addr(&full[s]), r & 1)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint64_t ad = umma_desc_sw128(smem_addr(sA + s * kGemmTileBytesA));
                const uint64_t bd = umma_desc_sw128(smem_addr(sB + s * kGemmTileBytesB));
#pragma unroll
                for (int k = 0; k < kGemmBK / 16; k++)  // 16 elements = 32 bytes = 2 units
                    umma_bf16(d, ad + 2 * k, bd + 2 * k, idesc, (kb | k) != 0);
                umma_commit(smem_addr(&empty[s]));
            }
            if (!ok) {
                *s_abort = 1u;
                atomicOr(a.status, kDevTimeout);
                break;
            }
            umma_commit(smem_addr(&accfull[acc]));
        }
    } else if (warp >= 2) {
        // ---- epilogue: warp w reads TMEM lanes 32*(w % 4) ..
        const int sub = warp & 3;
        int tc = 0;
        for (int t = blockIdx.x; t < total; t += gridDim.x, tc++) {
            const int acc = tc & 1, use = tc >> 1;
            // one decision for the whole warp: tcgen05.ld is warp-collective
            const bool ok = __all_sync(kFull, !*s_abort && mbar_wait(smem_addr(&accfull[acc]), use & 1));
            if (!ok) {
                if (lane == 0) {
                    *s_abort = 1u;
                    atomicOr(a.status, kDevTimeout);
                }
                break;
            }
            tc_fence_after();
            int e, m0, n0;
            gemm_tile(prefix, E, a.ntn, t, e, m0, n0);
            const int m = m0 + sub * 32 + lane;
            const bool valid = m < a.cnt[e];
            uint16_t *yrow = a.y + (a.eo[e] + m) * (int64_t)a.N + n0;
            const uint32_t taddr = tmem_base + ((uint32_t)(sub * 32) << 16) + (uint32_t)(acc * kGemmBN);
#pragma unroll 1
            for (int c = 0; c < kGemmBN / 16; c++) {
                uint32_t v[16];
                tmem_ld16(taddr + c * 16, v);
                if (valid) store_bf16x16(yrow + c * 16, v);
            }
            tc_fence_before();
            mbar_arrive(smem_addr(&accempty[acc]));
        }
    }
    // every MMA this block issued has finished before the TMEM is freed: a
    // last commit arrives on `drain` once they have (bounded wait)
    if (warp == 1 && lane == 0 && total > (int)blockIdx.x) {
        umma_commit(smem_addr(drain));
        if (!mbar_wait(smem_addr(drain), 0)) atomicOr(a.status, kDevTimeout);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                     "r"(2 * kGemmBN));
    }
}

// ---------------------------------------------------------------------------
// bf16 on CTA pairs: the two-CTA MMA (tcgen05.mma.cta_group::2, M = 256).
// A thread-block cluster of two CTAs on two SMs computes a 256-row x 256-column
// output tile: CTA r holds rows 128r .. 128r+127 of A and rows 128r .. of the
// tile's 256 weight rows (half of B), and its TMEM holds its 128 output rows.
// One instruction multiplies the pair's whole tile, each SM reading its own
// halves of A and B, so an SM reads half the B bytes per FLOP that a one-CTA
// 128 x 256 tile reads.
//
// Both CTAs load their halves with the pair form of TMA, whose bytes complete
// on the leader's (rank 0) stage barrier; the leader expects both CTAs' bytes
// and one thread of it issues the MMAs, committing each stage to both CTAs'
// empty barriers and each finished tile to both CTAs' accumulator barriers
// (multicast commit).  Each CTA's epilogue reads its own TMEM rows and
// arrives on the leader's accumulator-empty barrier (256 arrivals).  Waits
// are bounded as in the one-CTA kernels; the pair meets at a cluster barrier
// after its last MMA has completed and before either frees its TMEM.
// ---------------------------------------------------------------------------
constexpr int kG2Stages = 6;
constexpr int kG2Half = 128 * kGemmBK * 2;  // 16 KB: a CTA's half of an A or B K step
constexpr int kG2BM = 256, kG2BN = 256;

__host__ __device__ constexpr size_t gemm2_smem_bytes() {
    return 1024 + (size_t)kG2Stages * 2 * kG2Half + (2 * kG2Stages + 5) * 8 + 16 +
           (kGemmMaxExperts + 1) * 4 + 256;
}

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// shared::cluster address of the same variable in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t smem_in_rank(uint32_t saddr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
    return r;
}
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                     : "memory");
}
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
                 : "memory");
}
// this CTA's half of a K step, completing on the leader's barrier
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap *map, int c0,
                                                 int c1, uint32_t bar_cluster) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar_cluster)
        : "memory");
}
__device__ __forceinline__ void umma_bf16_pair(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                               uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// arrive on the barrier at this shared offset in both CTAs of the pair once
// the leader's MMAs issued so far have completed
__device__ __forceinline__ void umma_commit_pair(uint32_t bar) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
        " [%0], %1;" ::"r"(bar),
        "h"((uint16_t)0x3)
        : "memory");
}

__global__ void __launch_bounds__(kGemmThreads, 1)
    expert_gemm2_kernel(const __grid_constant__ CUtensorMap tm_a,
                        const __grid_constant__ CUtensorMap tm_b, GemmArgs a) {
    extern __shared__ uint8_t gsm_raw[];
    uint8_t *gsm = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(gsm_raw) + 1023) & ~(uintptr_t)1023);
    constexpr int S = kG2Stages;
    uint8_t *sA = gsm;
    uint8_t *sB = gsm + S * kG2Half;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sB + S * kG2Half);
    uint64_t *full = bars, *empty = bars + S;
    uint64_t *accfull = bars + 2 * S, *accempty = accfull + 2;
    uint64_t *drain = accempty + 2;
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(drain + 1);
    volatile uint32_t *s_abort = s_tmem + 1;
    int *prefix = reinterpret_cast<int *>(s_tmem + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const bool leader = rank == 0;
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    const int E = a.E;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; s++) {
            mbar_init(smem_addr(&full[s]), 1);   // the leader's expect_tx (bytes of both CTAs)
            mbar_init(smem_addr(&empty[s]), 1);  // the leader's multicast commit
        }
        for (int b = 0; b < 2; b++) {
            mbar_init(smem_addr(&accfull[b]), 1);
            mbar_init(smem_addr(&accempty[b]), 2 * 128);  // both CTAs' epilogue threads
        }
        mbar_init(smem_addr(drain), 1);
        *s_abort = 0u;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {  // both CTAs, same warp: 2 x 256 columns in each
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_addr(s_tmem)),
                     "r"(2 * kG2BN));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
    }
    pdl_enter();
    if (warp == 0) tile_prefix(prefix, E, a.cnt, a.ntn, lane, kG2BM);  // tiles of 256 rows
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();  // both CTAs' barriers initialised before any remote use
    tc_fence_after();
    const uint32_t tmem_base = *s_tmem;
    const int total = prefix[E];
    const int kblocks = a.H / kGemmBK;

    // tile t -> expert, first row (of the pair's 256) and first column
    auto tile = [&](int t, int &e, int &m0, int &n0) {
        int lo = 0, hi = E - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (prefix[mid] <= t) lo = mid;
            else hi = mid - 1;
        }
        e = lo;
        const int local = t - prefix[e];
        const int mt = (prefix[e + 1] - prefix[e]) / a.ntn;
        m0 = (local % mt) * kG2BM;
        n0 = (local / mt) * kG2BN;
    };

    if (warp == 0 && lane == 0) {
        // ---- this CTA's halves of A and B
        int it = 0;
        for (int t = pair; t < total && !*s_abort; t += npairs) {
            int e, m0, n0;
            tile(t, e, m0, n0);
            const int arow = (int)a.eo[e] + m0 + 128 * (int)rank;
            const int brow = e * a.N + n0 + 128 * (int)rank;
            for (int kb = 0; kb < kblocks; kb++, it++) {
                const int s = it % S, r = it / S;
                if (!mbar_wait(smem_addr(&empty[s]), (r & 1) ^ 1)) {
                    *s_abort = 1u;
                    atomicOr(a.status, kDevTimeout);
                    break;
                }
                const uint32_t fb = smem_addr(&full[s]);
                if (leader) mbar_expect_tx(fb, 2 * 2 * kG2Half);
                const uint32_t fl = smem_in_rank(fb, 0);
                tma_load_2d_pair(smem_addr(sA + s * kG2Half), &tm_a, kb * kGemmBK, arow, fl);
                tma_load_2d_pair(smem_addr(sB + s * kG2Half), &tm_b, kb * kGemmBK, brow, fl);
            }
        }
        if (leader)  // the pair's copies in flight land before the leader leaves
            for (int j = 0; j < S && j < it; j++) {
                const int i2 = it - 1 - j, s = i2 % S, r = i2 / S;
                if (!mbar_wait(smem_addr(&full[s]), r & 1)) atomicOr(a.status, kDevTimeout);
            }
    } else if (warp == 1 && lane == 0 && leader) {
        // ---- MMAs for the pair
        const uint32_t idesc = umma_idesc_bf16(kG2BM, kG2BN);
        int it = 0, tc = 0;
        for (int t = pair; t < total && !*s_abort; t += npairs, tc++) {
            const int acc = tc & 1, use = tc >> 1;
            if (!mbar_wait(smem_addr(&accempty[acc]), (use & 1) ^ 1)) {
                *s_abort = 1u;
                atomicOr(a.status, kDevTimeout);
                break;
            }
            tc_fence_after();
            const uint32_t d = tmem_base + (uint32_t)(acc * kG2BN);
            bool ok = true;
            for (int kb = 0; kb < kblocks; kb++, it++) {
                const int s = it % S, r = it / S;
                if (!mbar_wait(smem_addr(&full[s]), r & 1)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint64_t ad = umma_desc_sw128(smem_addr(sA + s * kG2Half));
                const uint64_t bd = umma_desc_sw128(smem_addr(sB + s * kG2Half));
#pragma unroll
                for (int k = 0; k < kGemmBK / 16; k++)
                    umma_bf16_pair(d, ad + 2 * k, bd + 2 * k, idesc, (kb | k) != 0);
                umma_commit_pair(smem_addr(&empty[s]));
            }
            if (!ok) {
                *s_abort = 1u;
                atomicOr(a.status, kDevTimeout);
                break;
            }
            umma_commit_pair(smem_addr(&accfull[acc]));
        }
    } else if (warp >= 2) {
        // ---- epilogue: this CTA's 128 rows of the pair's tile
        const int sub = warp & 3;
        const uint32_t empty_leader0 = smem_in_rank(smem_addr(&accempty[0]), 0);
        const uint32_t empty_leader1 = smem_in_rank(smem_addr(&accempty[1]), 0);
        int tc = 0;
        for (int t = pair; t < total; t += npairs, tc++) {
            const int acc = tc & 1, use = tc >> 1;
            const bool ok =
                __all_sync(kFull, !*s_abort && mbar_wait(smem_addr(&accfull[acc]), use & 1));
            if (!ok) {
                if (lane == 0) {
                    *s_abort = 1u;
                    atomicOr(a.status, kDevTimeout);
                }
                break;
            }
            tc_fence_after();
            int e, m0, n0;
            tile(t, e, m0, n0);
            const int m = m0 + 128 * (int)rank + sub * 32 + lane;
            const bool valid = m < a.cnt[e];
            uint16_t *yrow = a.y + (a.eo[e] + m) * (int64_t)a.N + n0;
            const uint32_t taddr =
                tmem_base + ((uint32_t)(sub * 32) << 16) + (uint32_t)(acc * kG2BN);
#pragma unroll 1
            for (int c = 0; c < kG2BN / 16; c++) {
                uint32_t v[16];
                tmem_ld16(taddr + c * 16, v);
                if (valid) store_bf16x16(yrow + c * 16, v);
            }
            tc_fence_before();
            mbar_arrive_remote(acc ? empty_leader1 : empty_leader0);
        }
    }
    // the leader's MMAs have all completed before either CTA frees its TMEM (a
    // commit to the leader's own barrier only)
    if (warp == 1 && lane == 0 && leader && total > pair) {
        asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                         smem_addr(drain))
                     : "memory");
        if (!mbar_wait(smem_addr(drain), 0)) atomicOr(a.status, kDevTimeout);
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                     "r"(2 * kG2BN));
    }
}

// ---------------------------------------------------------------------------
// MX operands: e4m3 (MXFP8) or packed e2m1 (MXFP4) codes with one e8m0 scale
// per 32 elements on both the received rows and the weights, multiplied by
// the block-scaled MMA: tcgen05.mma kind::mxf8f6f4.block_scale (e4m3, K = 32
// per instruction, one scale per row of A and of B) or kind::mxf4.block_scale
// .block32 (e2m1 two a byte, K = 64, two scales per row).
//
// A K step is 128 bytes of codes per row (one 128-byte swizzle row): 4
// instructions, 4 (MXFP8) or 8 (MXFP4) scale blocks.  The scales of a step
// are read from the rows' scale region by one gathering warp and written to
// shared memory in the arrangement that tcgen05.cp .32x128b.warpx4 copies to
// TMEM: per 128 rows and group of 4 scale blocks, a 512-byte chunk in which
// the 16 bytes of lane l hold rows l, l+32, l+64, l+96 (4 bytes each).  In
// TMEM row m's scale for block j of a group then sits in lane m % 32 (of
// every lane quarter), column (group's first) + m / 32, byte j; an
// instruction names the first of its blocks by the scale-factor id (byte j,
// also bits 30-31 of the scale address).
//
// Warps: 0 loads the code tiles with TMA; 1 allocates TMEM and one lane
// issues the scale copies and the MMAs; 2 gathers the scales; 3 - 6 run the
// epilogue.
//
// GLU = true (MXFP8 only) is the first layer of the experts' gated MLP
// ("[feat] A5 deep fused moe supported": GMM1, SwiGLU and Requant): the
// weights are [E][2I][K] with the gate projection in rows 0 .. I-1 and the up
// projection in rows I .. 2I-1 of each expert; a tile's B operand is BN/2
// gate rows j0 .. and the same BN/2 up rows (two TMA boxes), so the
// accumulator holds gate columns 0 .. BN/2-1 and the matching up columns
// BN/2 .. BN-1.  The epilogue forms z = silu(gate) * up in fp32 from the
// accumulator and writes it requantised to MXFP8 (one e8m0 scale per 32
// outputs, the dispatch's rule): codes [rows][I], scales [rows][I/32].  A stage is full when the TMA bytes have landed and the gathering
// warp has arrived.  TMEM holds kAcc accumulators of BN columns and the
// scales behind them: two accumulators (the epilogue of one tile overlaps the
// next tile's MMAs) where they and the scales fit in 512 columns, else one.
// TMEM scale columns: A's groups (4 columns each), then B's (group-major,
// then 128-row block).
// ---------------------------------------------------------------------------
constexpr int kMxBK = 128, kMxThreads = 224;
// K steps whose scale loads the gathering warp issues together (MXFP4 has
// twice the scale bytes a step: fewer steps keep its registers unspilled)
template <bool FP4>
__host__ __device__ constexpr int sf_group() { return FP4 ? 4 : 8; }
static_assert(sf_group<false>() % 4 == 0 && sf_group<true>() % 4 == 0,
              "16-byte scale loads cover four steps");

template <int BN, bool FP4, int BM = kGemmBM>
struct MxCfg {
    static constexpr int kNsf = FP4 ? 2 : 1;                // scale blocks per instruction
    static constexpr int kGroups = kNsf;                    // groups of 4 blocks per K step
    static constexpr int kChunksA = BM / 128;               // 128-row halves of A (M = 128 MMAs)
    static constexpr int kChunksB = (BN + 127) / 128;       // 128-row blocks of B
    static constexpr int kChunks = kChunksA + kChunksB;
    static constexpr int kSfCols = 4 * kGroups * kChunks;   // TMEM columns of the scales
    static constexpr int kAccCols = kChunksA * BN;          // one accumulator: BN columns a half
    static constexpr int kAcc = (2 * kAccCols + kSfCols <= 512) ? 2 : 1;
    static constexpr int kBytesA = BM * kMxBK;              // 16 KB a half
    static constexpr int kBytesB = BN * kMxBK;
    static constexpr int kSfBytes = 512 * kGroups * kChunks;  // a stage's scales, A then B
    static constexpr int kSfCol = kAcc * kAccCols;          // TMEM column of A's scales
    // Stages: as many as the shared memory holds (at most 8).  The operands
    // stream from L2 and DRAM at a latency of about a microsecond, so the
    // bytes in flight per SM, not the issue rate, set the narrow tiles' pace.
    static constexpr size_t kFixed = 1024 + 16 + (kGemmMaxExperts + 1) * 4 + 256 + 5 * 8;
    static constexpr int kStageBytes = kBytesA + kBytesB + kSfBytes;
    static constexpr int kStagesFit = (int)((227 * 1024 - kFixed) / (kStageBytes + 16));
    static constexpr int kStages = kStagesFit > 8 ? 8 : kStagesFit;
    static constexpr size_t smem() {
        return kFixed + (size_t)kStages * kStageBytes + (size_t)2 * kStages * 8;
    }
    static_assert(kStages >= (BM == 128 ? 4 : 3), "pipeline depth");
    static_assert(BN % 32 == 0 && BN >= 64 && BN <= 256, "N tile");
    static_assert(BM == 128 || BM == 256, "M tile");
    static_assert(kAcc * kAccCols + kSfCols <= 512, "TMEM columns");
};

struct MxArgs {
    int E, K, N;             // experts, depth (elements of a row), output columns
    int ntn;                 // N / BN (GLU: I / (BN/2))
    int I;                   // GLU: the intermediate size (N = 2I)
    int64_t rows;            // rows of the receive buffer (scale rows that exist)
    const int64_t *eo;       // [E+1] first row of each expert (packed layout)
    const int64_t *cnt;      // [E] rows of each expert
    const uint8_t *xs;       // [rows][K/32] e8m0 scales of the received rows
    const uint8_t *ws;       // [E*N][K/32] e8m0 scales of the weights
    uint16_t *y;             // [rows][N] bf16 (not GLU)
    uint8_t *zc;             // GLU: [rows][I] e4m3 codes of the requantised z
    uint8_t *zs;             // GLU: [rows][I/32] their e8m0 scales
    uint32_t *status;
};

// silu(g) * u in fp32: g / (1 + e^-g) with the library's expf and
// correctly rounded division and multiply (a very negative g gives
// e^-g = inf and silu = -0)
__device__ __forceinline__ float swiglu(float g, float u) {
    return __fmul_rn(__fdiv_rn(g, __fadd_rn(1.0f, expf(-g))), u);
}

// instruction descriptor of the block-scaled MMA: A and B formats (e4m3 = 0
// for kind::mxf8f6f4, e2m1 = 1 for kind::mxf4), both K-major, e8m0 scales,
// N, M (the scale-factor ids are or-ed in per instruction)
__host__ __device__ constexpr uint32_t umma_idesc_mx(int M, int N, bool fp4) {
    return (fp4 ? (1u << 7) | (1u << 10) : 0u) | ((uint32_t)(N >> 3) << 17) | (1u << 23) |
           ((uint32_t)(M >> 4) << 24);
}
template <bool FP4>
__device__ __forceinline__ void umma_mx(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                        uint32_t idesc, uint32_t tsfa, uint32_t tsfb,
                                        uint32_t accumulate) {
    if constexpr (FP4)
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %6, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%4], [%5], p;\n\t}"
            ::"r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(tsfa), "r"(tsfb), "r"(accumulate)
            : "memory");
    else
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %6, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%4], [%5], p;\n\t}"
            ::"r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(tsfa), "r"(tsfb), "r"(accumulate)
            : "memory");
}
// shared-memory descriptor of 32 rows x 16 bytes, rows 16 bytes apart (no
// swizzle, K-major: 8-row core matrices of 128 contiguous bytes, 128 bytes
// between them)
__device__ __forceinline__ uint64_t sf_desc(uint32_t saddr) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)8 << 32) | ((uint64_t)1 << 46);
}
__device__ __forceinline__ void tmem_cp_32x128b_x4(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc)
                 : "memory");
}
__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
                 "r"(d)
                 : "memory");
}

// 128-row halves of a row tile that hold rows of the expert: a 256-row tile
// whose upper half would hold none is loaded, multiplied and stored as a
// 128-row tile (no more MMA work than 128-row tiles at the expert's end)
template <int HA>
__device__ __forceinline__ int tile_halves(int64_t cnt, int m0) {
    return (HA > 1 && cnt - m0 > 128) ? 2 : 1;
}

template <int BN, bool FP4, bool GLU = false, int BM = kGemmBM>
__global__ void __launch_bounds__(kMxThreads, 1)
    expert_gemm_mx_kernel(const __grid_constant__ CUtensorMap tm_a,
                          const __grid_constant__ CUtensorMap tm_b, MxArgs a) {
    using C = MxCfg<BN, FP4, BM>;
    static_assert(!GLU || (!FP4 && BN % 64 == 0), "GLU: MXFP8, whole 32-blocks per half tile");
    static_assert(!GLU || BM == 128, "GLU: 128-row tiles");
    constexpr int HA = C::kChunksA;  // 128-row halves of a row tile (one M = 128 MMA each)
    constexpr int TN = GLU ? BN / 2 : BN;  // output columns a tile advances by
    constexpr int S = C::kStages;
    extern __shared__ uint8_t gsm_raw[];
    uint8_t *gsm = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(gsm_raw) + 1023) & ~(uintptr_t)1023);
    uint8_t *sA = gsm;
    uint8_t *sB = sA + S * C::kBytesA;
    uint8_t *sSF = sB + S * C::kBytesB;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sSF + S * C::kSfBytes);
    uint64_t *full = bars, *empty = bars + S;
    uint64_t *accfull = bars + 2 * S, *accempty = accfull + 2;
    uint64_t *drain = accempty + 2;
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(drain + 1);
    volatile uint32_t *s_abort = s_tmem + 1;
    int *prefix = reinterpret_cast<int *>(s_tmem + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int E = a.E;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; s++) {
            mbar_init(smem_addr(&full[s]), 2);  // the TMA bytes' arrival + the scale warp's
            mbar_init(smem_addr(&empty[s]), 1);
        }
        for (int b = 0; b < 2; b++) {
            mbar_init(smem_addr(&accfull[b]), 1);
            mbar_init(smem_addr(&accempty[b]), 128);
        }
        mbar_init(smem_addr(drain), 1);
        *s_abort = 0u;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {  // the whole warp: all 512 columns (accumulators, then the scales)
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_addr(s_tmem)),
                     "r"(512));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    pdl_enter();
    if (warp == 0) tile_prefix(prefix, E, a.cnt, a.ntn, lane, BM);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *s_tmem;
    const int total = prefix[E];
    const int kblocks = (FP4 ? a.K / 2 : a.K) / kMxBK;  // 128-byte K steps

    if (warp == 0 && lane == 0) {
        // ---- code tiles
        int it = 0;
        for (int t = blockIdx.x; t < total && !*s_abort; t += gridDim.x) {
            int e, m0, n0;
            gemm_tile(prefix, E, a.ntn, t, e, m0, n0, TN, BM);
            const int arow = (int)a.eo[e] + m0, brow = e * a.N + n0;
            const int halves = tile_halves<HA>(a.cnt[e], m0);
            for (int kb = 0; kb < kblocks; kb++, it++) {
                const int s = it % S, r = it / S;
                if (!mbar_wait(smem_addr(&empty[s]), (r & 1) ^ 1)) {
                    *s_abort = 1u;
                    atomicOr(a.status, kDevTimeout);
                    break;
                }
                const uint32_t fb = smem_addr(&full[s]);
                mbar_expect_tx(fb, halves * 128 * kMxBK + C::kBytesB);
                for (int h = 0; h < halves; h++)
                    tma_load_2d(smem_addr(sA + s * C::kBytesA + h * 128 * kMxBK), &tm_a, kb * kMxBK,
                                arow + 128 * h, fb);
                if constexpr (GLU) {  // gate rows, then the same rows of the up projection
                    tma_load_2d(smem_addr(sB + s * C::kBytesB), &tm_b, kb * kMxBK, brow, fb);
                    tma_load_2d(smem_addr(sB + s * C::kBytesB + TN * kMxBK), &tm_b, kb * kMxBK,
                                brow + a.I, fb);
                } else {
                    tma_load_2d(smem_addr(sB + s * C::kBytesB), &tm_b, kb * kMxBK, brow, fb);
                }
            }
        }
        for (int j = 0; j < S && j < it; j++) {  // copies in flight land before leaving
            const int i2 = it - 1 - j, s = i2 % S, r = i2 / S;
            if (!mbar_wait(smem_addr(&full[s]), r & 1)) atomicOr(a.status, kDevTimeout);
        }
    } else if (warp == 1 && lane == 0) {
        // ---- scale copies and MMAs
        const uint32_t idesc = umma_idesc_mx(kGemmBM, BN, FP4);
        const uint32_t tsfa = tmem_base + (uint32_t)C::kSfCol, tsfb = tsfa + 4 * C::kGroups * HA;
        int it = 0, tc = 0;
        for (int t = blockIdx.x; t < total && !*s_abort; t += gridDim.x, tc++) {
            const int acc = tc % C::kAcc, use = tc / C::kAcc;
            if (!mbar_wait(smem_addr(&accempty[acc]), (use & 1) ^ 1)) {
                *s_abort = 1u;
                atomicOr(a.status, kDevTimeout);
                break;
            }
            tc_fence_after();
            const uint32_t d = tmem_base + (uint32_t)(acc * C::kAccCols);
            int halves = 1;
            if constexpr (HA > 1) {
                int e, m0, n0;
                gemm_tile(prefix, E, a.ntn, t, e, m0, n0, TN, BM);
                halves = tile_halves<HA>(a.cnt[e], m0);
            }
            bool ok = true;
            for (int kb = 0; kb < kblocks; kb++, it++) {
                const int s = it % S, r = it / S;
                if (!mbar_wait(smem_addr(&full[s]), r & 1)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t sf = smem_addr(sSF + s * C::kSfBytes);
#pragma unroll
                for (int c = 0; c < C::kGroups * C::kChunks; c++)  // A's, then B's
                    tmem_cp_32x128b_x4(tsfa + 4 * c, sf_desc(sf + 512 * c));
                const uint64_t bd = umma_desc_sw128(smem_addr(sB + s * C::kBytesB));
#pragma unroll
                for (int k = 0; k < 4; k++) {  // 32 bytes of codes = 2 units each
                    const int blk = k * C::kNsf, grp = blk / 4;
                    const uint32_t byte = (uint32_t)(blk % 4);
#pragma unroll
                    for (int h = 0; h < HA; h++) {  // the halves share the stage's B tile
                        if (h >= halves) break;
                        const uint64_t ad =
                            umma_desc_sw128(smem_addr(sA + s * C::kBytesA + h * 128 * kMxBK));
                        umma_mx<FP4>(d + h * BN, ad + 2 * k, bd + 2 * k,
                                     idesc | (byte << 29) | (byte << 4),
                                     (tsfa + 4 * (grp * HA + h)) | (byte << 30),
                                     (tsfb + 4 * C::kChunksB * grp) | (byte << 30), (kb | k) != 0);
                    }
                }
                umma_commit(smem_addr(&empty[s]));
            }
            if (!ok) {
                *s_abort = 1u;
                atomicOr(a.status, kDevTimeout);
                break;
            }
            umma_commit(smem_addr(&accfull[acc]));
        }
    } else if (warp == 2) {
        // ---- scales: 4 bytes (one K step) of every row of the A and B tiles
        // The loads of sf_group() K steps are issued together: one step's
        // loads would leave a whole L2 latency between consecutive steps.
        constexpr int G = sf_group<FP4>();
        const int SB = a.K / 32;
        // 16-byte loads where every row's scales start on a 16-byte boundary
        // (the scale regions themselves are 16-byte aligned)
        const bool vec = SB % 16 == 0;
        int it = 0;
        for (int t = blockIdx.x; t < total; t += gridDim.x) {
            if (__shfl_sync(kFull, (int)*s_abort, 0)) break;
            int e, m0, n0;
            gemm_tile(prefix, E, a.ntn, t, e, m0, n0, TN, BM);
            const int64_t arow0 = a.eo[e] + m0;
            const int64_t brow0 = (int64_t)e * a.N + n0;
            // weight row of B-tile row n (GLU: the up rows follow the gate rows)
            auto brow_of = [&](int n) -> int64_t {
                return GLU ? brow0 + n + (n >= TN ? (int64_t)a.I - TN : 0) : brow0 + n;
            };
            bool ok = true;
            for (int kb0 = 0; kb0 < kblocks && ok; kb0 += G) {
                const int g = min(G, kblocks - kb0);
                constexpr int NG = C::kGroups;
                uint32_t va[G][NG][HA][4], vb[G][NG][C::kChunksB][4];
                if (vec && g == G) {
                    // a row's scales of the G steps are G * NG contiguous words,
                    // 16-byte aligned: G * NG / 4 16-byte loads per row
#pragma unroll
                    for (int ha = 0; ha < HA; ha++)
#pragma unroll
                    for (int j = 0; j < 4; j++) {
                        const int64_t row = arow0 + 128 * ha + lane + 32 * j;
#pragma unroll
                        for (int h = 0; h < G * NG / 4; h++) {
                            const uint4 w4 = row < a.rows
                                                 ? __ldg(reinterpret_cast<const uint4 *>(
                                                       a.xs + row * SB + kb0 * NG * 4) + h)
                                                 : make_uint4(0u, 0u, 0u, 0u);
                            const uint32_t wv[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
                            for (int u = 0; u < 4; u++)
                                va[(4 * h + u) / NG][(4 * h + u) % NG][ha][j] = wv[u];
                        }
                    }
#pragma unroll
                    for (int c = 0; c < C::kChunksB; c++)
#pragma unroll
                        for (int j = 0; j < 4; j++) {
                            const int n = 128 * c + 32 * j + lane;
#pragma unroll
                            for (int h = 0; h < G * NG / 4; h++) {
                                const uint4 w4 = n < BN ? __ldg(reinterpret_cast<const uint4 *>(
                                                              a.ws + brow_of(n) * SB + kb0 * NG * 4) + h)
                                                        : make_uint4(0u, 0u, 0u, 0u);
                                const uint32_t wv[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
                                for (int u = 0; u < 4; u++)
                                    vb[(4 * h + u) / NG][(4 * h + u) % NG][c][j] = wv[u];
                            }
                        }
                } else {
#pragma unroll
                for (int q = 0; q < G; q++) {
                    if (q >= g) break;
                    const int kb = kb0 + q;
#pragma unroll
                    for (int gg = 0; gg < NG; gg++) {
                        const int off = (kb * NG + gg) * 4;  // the group's 4 scale bytes
#pragma unroll
                        for (int ha = 0; ha < HA; ha++)
#pragma unroll
                        for (int j = 0; j < 4; j++) {
                            const int64_t row = arow0 + 128 * ha + lane + 32 * j;
                            va[q][gg][ha][j] = row < a.rows ? __ldg(reinterpret_cast<const uint32_t *>(
                                                                  a.xs + row * SB + off))
                                                            : 0u;
                        }
#pragma unroll
                        for (int c = 0; c < C::kChunksB; c++)
#pragma unroll
                            for (int j = 0; j < 4; j++) {
                                const int n = 128 * c + 32 * j + lane;
                                vb[q][gg][c][j] = n < BN ? __ldg(reinterpret_cast<const uint32_t *>(
                                                               a.ws + brow_of(n) * SB + off))
                                                         : 0u;
                            }
                    }
                }
                }
#pragma unroll
                for (int q = 0; q < G; q++) {
                    if (q >= g) break;
                    const int s = it % S, r = it / S;
                    int got = 1;
                    if (lane == 0) got = mbar_wait(smem_addr(&empty[s]), (r & 1) ^ 1);
                    if (!__shfl_sync(kFull, got, 0)) {
                        ok = false;
                        break;
                    }
                    const uint32_t st = smem_addr(sSF + s * C::kSfBytes) + lane * 16;
#pragma unroll
                    for (int gg = 0; gg < NG; gg++) {
#pragma unroll
                        for (int ha = 0; ha < HA; ha++)
                            st_shared_v4(st + 512 * (gg * HA + ha), va[q][gg][ha][0],
                                         va[q][gg][ha][1], va[q][gg][ha][2], va[q][gg][ha][3]);
#pragma unroll
                        for (int c = 0; c < C::kChunksB; c++)
                            st_shared_v4(st + 512 * (NG * HA + gg * C::kChunksB + c),
                                         vb[q][gg][c][0], vb[q][gg][c][1], vb[q][gg][c][2],
                                         vb[q][gg][c][3]);
                    }
                    // the copies to TMEM read shared memory through the async proxy
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    __syncwarp();
                    if (lane == 0) mbar_arrive(smem_addr(&full[s]));
                    it++;
                }
            }
            if (!ok) {
                if (lane == 0) {
                    *s_abort = 1u;
                    atomicOr(a.status, kDevTimeout);
                }
                break;
            }
        }
    } else if (warp >= 3) {
        // ---- epilogue: warp w reads TMEM lanes 32*(w % 4) ..
        const int sub = warp & 3;
        int tc = 0;
        for (int t = blockIdx.x; t < total; t += gridDim.x, tc++) {
            const int acc = tc % C::kAcc, use = tc / C::kAcc;
            const bool ok =
                __all_sync(kFull, !*s_abort && mbar_wait(smem_addr(&accfull[acc]), use & 1));
            if (!ok) {
                if (lane == 0) {
                    *s_abort = 1u;
                    atomicOr(a.status, kDevTimeout);
                }
                break;
            }
            tc_fence_after();
            int e, m0, n0;
            gemm_tile(prefix, E, a.ntn, t, e, m0, n0, TN, BM);
#pragma unroll 1
            for (int ha = 0; ha < tile_halves<HA>(a.cnt[e], m0); ha++) {  // the tile's row halves
                const int m = m0 + 128 * ha + sub * 32 + lane;
                const bool valid = m < a.cnt[e];
                const uint32_t taddr = tmem_base + ((uint32_t)(sub * 32) << 16) +
                                       (uint32_t)(acc * C::kAccCols + ha * BN);
                if constexpr (GLU) {
                    const int64_t row = a.eo[e] + m;
                    uint8_t *zrow = a.zc + row * (int64_t)a.I + n0;
                    uint8_t *zsrow = a.zs + row * (int64_t)(a.I / 32) + n0 / 32;
#pragma unroll 1
                    for (int c = 0; c < TN / 32; c++) {  // one MX block of 32 outputs
                        uint32_t g0[16], g1[16], u0[16], u1[16];
                        tmem_ld16(taddr + c * 32, g0);
                        tmem_ld16(taddr + c * 32 + 16, g1);
                        tmem_ld16(taddr + TN + c * 32, u0);
                        tmem_ld16(taddr + TN + c * 32 + 16, u1);
                        float z[32];
                        float amax = 0.0f;
#pragma unroll
                        for (int i = 0; i < 16; i++) {
                            z[i] = swiglu(__uint_as_float(g0[i]), __uint_as_float(u0[i]));
                            z[16 + i] = swiglu(__uint_as_float(g1[i]), __uint_as_float(u1[i]));
                            amax = fmaxf(amax, fmaxf(fabsf(z[i]), fabsf(z[16 + i])));
                        }
                        const int X = mx_exponent_fast<448>(amax);
                        const float mult = exp2_neg(X);
                        uint32_t w[8];
#pragma unroll
                        for (int q = 0; q < 8; q++)
                            w[q] = cvt_e4m3x2(__fmul_rn(z[4 * q], mult),
                                              __fmul_rn(z[4 * q + 1], mult)) |
                                   (cvt_e4m3x2(__fmul_rn(z[4 * q + 2], mult),
                                               __fmul_rn(z[4 * q + 3], mult))
                                    << 16);
                        if (valid) {
                            st_v4(zrow + c * 32, make_uint4(w[0], w[1], w[2], w[3]));
                            st_v4(zrow + c * 32 + 16, make_uint4(w[4], w[5], w[6], w[7]));
                            zsrow[c] = (uint8_t)(X + 127);
                        }
                    }
                } else {
                    uint16_t *yrow = a.y + (a.eo[e] + m) * (int64_t)a.N + n0;
                    static_assert(BN % 32 == 0, "32-column epilogue steps");
#pragma unroll 1
                    for (int c = 0; c < BN / 32; c++) {  // 32 columns a TMEM load
                        uint32_t v[32];
                        tmem_ld32(taddr + c * 32, v);
                        if (valid) {
                            store_bf16x16(yrow + c * 32,
                                          *reinterpret_cast<const uint32_t(*)[16]>(v));
                            store_bf16x16(yrow + c * 32 + 16,
                                          *reinterpret_cast<const uint32_t(*)[16]>(v + 16));
                        }
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(smem_addr(&accempty[acc]));
        }
    }
    if (warp == 1 && lane == 0 && total > (int)blockIdx.x) {
        umma_commit(smem_addr(drain));
        if (!mbar_wait(smem_addr(drain), 0)) atomicOr(a.status, kDevTimeout);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                     "r"(512));
    }
}

}  // namespace ep
