// Grouped, persistent, warp-specialised bf16 GEMM on the 5th-generation tensor cores
// (tcgen05 + TMEM + TMA) for the three products of one Newton-Schulz iteration
// ("Muon优化器" page, section "Newton-Schulz 迭代": A = X X^T, B = bA + cA^2, X = aX + BX).
//
// Two CTAs of a cluster (a pair on two SMs) compute one 256 x 256 output tile with
// tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 16): each CTA stages its 128 rows of A
// and its 128 columns of B, so every SM reads half of B's bytes a 1-SM 128 x 256 tile
// would; each CTA's TMEM holds its 128 rows x 256 fp32 columns, twice (double buffer).
// Roles per CTA (384 threads):
//   warp 0 lane 0 : TMA producer -- kTcStages-deep ring of (128 x 64 A, 128 x 64 B) bf16 tiles,
//                   128-byte swizzled, K-major or MN-major per problem; the loads of both
//                   CTAs count on the leader CTA's "full" barrier (.cta_group::2 form)
//   warp 1 lane 0 : MMA issuer (leader CTA only) -- commits free the stage in both CTAs
//                   and signal both CTAs' epilogues (commit with a CTA mask)
//   warp 2        : TMEM allocation / release (pair-wide)
//   warps 4..11   : epilogue -- tcgen05.ld of its 32-lane quarter and half of the columns,
//                   alpha/beta/scale in fp32, bf16 (hi, lo) stores, mirrored stores for
//                   symmetric outputs, then an arrival on the leader's "TMEM empty" barrier
// No TMA load uses cluster multicast.  Tiles of all problems of a stage come from one list;
// pair p takes tiles p, p + pairs, ...  Every wait is bounded (ptx_sm100.cuh).
#include <cstdio>

#include "kernels.cuh"
#include "ptx_sm100.cuh"

namespace muon {
namespace {

constexpr int BM = kTcBM, BN = kTcBN, BK = kTcBK, STAGES = kTcStages;
constexpr int HM = BM / 2, HN = BN / 2;              // per-CTA rows of A / columns of B
constexpr int A_BYTES = HM * BK * 2;                 // 16 KB
constexpr int B_BYTES = HN * BK * 2;                 // 16 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;       // per CTA
constexpr int PAIR_STAGE_BYTES = 2 * STAGE_BYTES;    // counted on the leader's barrier
constexpr int MN_CHUNK_BYTES = 64 * BK * 2;          // one 64(MN) x 64(K) box: 8 KB
constexpr int TMEM_COLS = 512;
constexpr int ACC_COLS = 256;
constexpr int BAR_BYTES = 256;
// Per epilogue warp, 32 x 32 bf16 chunks (64-byte rows): one for the direct store, one for the
// transposed mirror, and two for E (the chunk in use and the one being fetched).
constexpr int STG_BYTES = 32 * 64;
constexpr int STG_WARP_BYTES = 4 * STG_BYTES;
constexpr int SMEM_TOTAL = STAGES * STAGE_BYTES + BAR_BYTES + (kTcEpilogueThreads / 32) * STG_WARP_BYTES + 1024;
static_assert(SMEM_TOTAL <= 232448, "dynamic shared memory above the 227 KB per-CTA limit");
static_assert(HM == 128 && HN == 128, "pair tile is 256 x 256");

struct TileInfo {
    int p, m0, n0;
};
__device__ __forceinline__ TileInfo decode(uint32_t code) {
    TileInfo t;
    t.p = static_cast<int>(code >> 20);
    t.m0 = static_cast<int>((code >> 10) & 1023u) * BM;
    t.n0 = static_cast<int>(code & 1023u) * BN;
    return t;
}

__device__ __forceinline__ void segment_planes(const TcProblem& P, int seg, int& pa, int& pb) {
    const uint32_t c = (P.segs >> (4 * seg)) & 0xFu;
    pa = static_cast<int>(c & 3u);
    pb = static_cast<int>(c >> 2);
}

// Byte offset of 16-byte segment `seg` (0..3) of row `row` in a 32 x 64-byte staging chunk,
// segments XOR-swizzled by (row >> 1) & 3: a warp touching one segment of 32 rows, or 4
// segments of 8 rows, hits every bank group once per 8 lanes (no conflicts).
__device__ __forceinline__ int stg_off64(int row, int seg) { return row * 64 + 16 * (seg ^ ((row >> 1) & 3)); }

// 16-byte global -> shared copy (cp.async, L2 only); bytes past src_bytes are zero-filled.
__device__ __forceinline__ void cp_async16_zfill(void* smem_dst, const void* gmem_src, int src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(smem_dst)), "l"(gmem_src),
                 "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait_group() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// Transpose one 32 x 32 bf16 chunk held in staging layout (row r, 16-byte segment s at
// stg_off64(r, s)) into `dst` in the same layout: dst row c, column r = src row r, column c.
// Per column strip j, ldmatrix.trans reads the four 8 x 8 blocks (rows 8i.., segment j) of
// the strip and hands each lane its pieces of their transposes; stmatrix writes them as the
// blocks (rows 8j.., segment i) of dst.  Lane L addresses row L of src (ldmatrix: lanes
// 8i..8i+7 give block i's rows) and row 8j + (L & 7), segment L >> 3 of dst.  Both sides hit
// each bank group once per 8 rows.
__device__ __forceinline__ void stg_transpose32(const uint8_t* src, uint8_t* dst, int lane) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        uint32_t r0, r1, r2, r3;
        asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                     : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                     : "r"(smem_u32(src + stg_off64(lane, j)))
                     : "memory");
        asm volatile("stmatrix.sync.aligned.m8n8.x4.shared.b16 [%0], {%1, %2, %3, %4};"
                     ::"r"(smem_u32(dst + stg_off64(8 * j + (lane & 7), lane >> 3))), "r"(r0), "r"(r1), "r"(r2), "r"(r3)
                     : "memory");
    }
}

__device__ __forceinline__ void store_bf16x8(__nv_bfloat16* dst, const float* v) {
    uint4 w;
    w.x = pack_bf16x2(v[0], v[1]);
    w.y = pack_bf16x2(v[2], v[3]);
    w.z = pack_bf16x2(v[4], v[5]);
    w.w = pack_bf16x2(v[6], v[7]);
    *reinterpret_cast<uint4*>(dst) = w;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kTcThreads, 1)
tc_gemm_kernel(const TcProblem* __restrict__ probs, const uint32_t* __restrict__ tiles, int num_tiles,
               unsigned* dev_status) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
    uint64_t* full_bar = bars;                  // leader: TMA bytes of both CTAs landed
    uint64_t* empty_bar = bars + STAGES;        // both: MMAs reading the stage are done
    uint64_t* tfull_bar = bars + 2 * STAGES;    // both: accumulator ready
    uint64_t* tempty_bar = bars + 2 * STAGES + 2;   // leader: both epilogues drained it
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 4);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    // Programmatic dependent launch: the next launch of the chain may be scheduled as this
    // grid's CTAs finish (its prologue then overlaps this grid's tail).  It reads and writes
    // global data only after its own grid-dependency wait below.
    griddep_launch_dependents();
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();   // 0 = leader, 1 = peer
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull_bar[a], 1);
            mbar_init(&tempty_bar[a], 2 * kTcEpilogueThreads);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 2) {
        tmem_alloc_pair(tmem_slot, TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync();     // barriers of both CTAs initialised before any remote access
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // Leader-CTA addresses (shared::cluster window) of the barriers both CTAs signal.
    const uint32_t full_leader = mapa_shared(smem_u32(full_bar), 0);
    const uint32_t tempty_leader = mapa_shared(smem_u32(tempty_bar), 0);

    if (warp == 0 && lane == 0) {
        // ------------------------------------------------------------ TMA producer
        griddep_wait();   // operands written by the previous launch are complete and visible
        uint32_t stage = 0, phase = 0;
        int last_p = -1;
        bool ok = true;
        int issued_parity[STAGES];
#pragma unroll
        for (int s = 0; s < STAGES; ++s) issued_parity[s] = -1;
        for (int t = pair; t < num_tiles && ok; t += npairs) {
            const TileInfo ti = decode(tiles[t]);
            const TcProblem& P = probs[ti.p];
            if (ti.p != last_p) {
                for (int i = 0; i < kTcMaxPlanes; ++i) {
                    if (P.tmA[i]) tmap_acquire(P.tmA[i]);
                    if (P.tmB[i]) tmap_acquire(P.tmB[i]);
                }
                last_p = ti.p;
            }
            const bool a_mn = (P.flags & kProbAMn) != 0;
            const bool b_mn = (P.flags & kProbBMn) != 0;
            const int am0 = ti.m0 + HM * static_cast<int>(rank);
            const int bn0 = ti.n0 + HN * static_cast<int>(rank);
            const int kblocks = (P.K + BK - 1) / BK;
            const int nseg = P.nseg;
            for (int seg = 0; seg < nseg && ok; ++seg) {
                int pa, pb;
                segment_planes(P, seg, pa, pb);
                const CUtensorMap* ta = P.tmA[pa];
                const CUtensorMap* tb = P.tmB[pb];
                for (int kb = 0; kb < kblocks; ++kb) {
                    if (!mbar_wait(&empty_bar[stage], phase ^ 1u, abort_flag, dev_status)) { ok = false; break; }
                    uint8_t* sa = smem + stage * STAGE_BYTES;
                    uint8_t* sb = sa + A_BYTES;
                    const int k0 = P.k_begin + kb * BK;
                    const uint32_t fb = full_leader + stage * 8u;
                    if (rank == 0) {
                        mbar_arrive_expect_tx(&full_bar[stage], PAIR_STAGE_BYTES);
                        issued_parity[stage] = static_cast<int>(phase);
                    }
                    if (!a_mn) {
                        tma_load_2d_pair(sa, ta, fb, k0, am0);
                    } else {
#pragma unroll
                        for (int c = 0; c < HM / 64; ++c)
                            tma_load_2d_pair(sa + c * MN_CHUNK_BYTES, ta, fb, am0 + 64 * c, k0);
                    }
                    if (!b_mn) {
                        tma_load_2d_pair(sb, tb, fb, k0, bn0);
                    } else {
#pragma unroll
                        for (int c = 0; c < HN / 64; ++c)
                            tma_load_2d_pair(sb + c * MN_CHUNK_BYTES, tb, fb, bn0 + 64 * c, k0);
                    }
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
            }
        }
        if (!ok && rank == 0) {
            // Let copies already issued land before the pair exits (bounded).
            for (int s = 0; s < STAGES; ++s) {
                if (issued_parity[s] < 0) continue;
                const unsigned long long t0 = global_ns();
                bool landed = false;
                while (!(landed = mbar_try_wait(&full_bar[s], static_cast<uint32_t>(issued_parity[s]))) &&
                       global_ns() - t0 < 100000000ull) {
                }
                if (!landed) atomicOr(dev_status, kDevErrUndrained);
            }
        }
    } else if (warp == 1 && lane == 0 && rank == 0) {
        // ------------------------------------------------------------ MMA issuer (leader)
        uint32_t stage = 0, phase = 0, acc = 0, acc_phase = 0;
        bool ok = true;
        for (int t = pair; t < num_tiles && ok; t += npairs) {
            const TileInfo ti = decode(tiles[t]);
            const TcProblem& P = probs[ti.p];
            const bool a_mn = (P.flags & kProbAMn) != 0;
            const bool b_mn = (P.flags & kProbBMn) != 0;
            const uint32_t idesc = idesc_bf16_f32(BM, BN, a_mn, b_mn);
            const int kblocks = (P.K + BK - 1) / BK;
            const int nseg = P.nseg;
            if (!mbar_wait(&tempty_bar[acc], acc_phase ^ 1u, abort_flag, dev_status)) { ok = false; break; }
            tc_fence_after();
            const uint32_t d_tmem = tmem_base + acc * ACC_COLS;
            uint32_t accumulate = 0;
            for (int seg = 0; seg < nseg && ok; ++seg) {
                for (int kb = 0; kb < kblocks; ++kb) {
                    if (!mbar_wait(&full_bar[stage], phase, abort_flag, dev_status)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t base_a = smem_u32(smem + stage * STAGE_BYTES);
                    const uint32_t base_b = base_a + A_BYTES;
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k) {
                        const uint64_t ad = a_mn ? smem_desc_sw128(base_a + k * 2048, MN_CHUNK_BYTES, 1024)
                                                 : smem_desc_sw128(base_a + k * 32, 16, 1024);
                        const uint64_t bd = b_mn ? smem_desc_sw128(base_b + k * 2048, MN_CHUNK_BYTES, 1024)
                                                 : smem_desc_sw128(base_b + k * 32, 16, 1024);
                        tc_mma_bf16_pair(d_tmem, ad, bd, idesc, accumulate);
                        accumulate = 1;
                    }
                    tc_commit_pair(&empty_bar[stage], 0x3);
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
            }
            tc_commit_pair(&tfull_bar[acc], 0x3);
            if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
        }
        if (!ok) {
            // Drain: wait (bounded) until every MMA issued so far has finished.
            tc_commit_pair(&tfull_bar[acc], 0x3);
            const unsigned long long t0 = global_ns();
            bool done = false;
            while (!(done = mbar_try_wait(&tfull_bar[acc], acc_phase)) && global_ns() - t0 < 100000000ull) {
            }
            if (!done) atomicOr(dev_status, kDevErrUndrained);
        }
    } else if (warp >= 4) {
        // ------------------------------------------------------------ epilogue
        // 8 warps: warp & 3 selects the TMEM lane quarter (rows), (warp - 4) >> 2 the half of
        // the 256 columns.  tcgen05.ld gives lane L row L of a 32 x 32 chunk.  For bf16 E and
        // outputs every global access is coalesced: E is fetched as 8 rows x 64 B per
        // instruction and turned into rows through this warp's staging buffer, results go back
        // through it and out as 8 rows x 64 B per instruction, and the mirror of a symmetric
        // output is transposed there.  (A lane-per-row access touches 32 lines per instruction;
        // measured on the Llama-7B set, that traffic alone lowered the power-capped clock from
        // 1.94 to 1.46 GHz.)  fp32 problems and chunks on the diagonal of a symmetric output
        // keep per-lane accesses (the diagonal needs per-element masks).  E is prefetched one
        // chunk ahead, the first chunk before the accumulator wait.
        const int q = warp & 3;
        const int c_beg = ((warp - 4) >> 2) * (BN / 64);
        const int c_end = c_beg + BN / 64;
        uint8_t* stg = smem + STAGES * STAGE_BYTES + BAR_BYTES + (warp - 4) * STG_WARP_BYTES;   // direct stores
        uint8_t* stg_t = stg + STG_BYTES;              // transposed chunk of a mirror store
        uint8_t* stg_e = stg + 2 * STG_BYTES;          // E of two chunks (double buffer)
        const int crow = lane >> 2, cseg = lane & 3;   // coalesced layout: rows crow + 8i, segment cseg
        griddep_wait();   // E, the scale and the outputs' previous readers are done
        uint32_t acc = 0, acc_phase = 0;
        for (int t = pair; t < num_tiles; t += npairs) {
            const TileInfo ti = decode(tiles[t]);
            const TcProblem& P = probs[ti.p];
            float f = 1.0f;
            if (P.dscale != nullptr && P.scale_pow > 0) {
                const float s = __ldg(P.dscale);
                f = (P.scale_pow == 1) ? s : s * s;
            }
            const float alpha = P.alpha * f;
            const float beta = P.beta * f;
            const bool sym = (P.flags & kProbSym) != 0;
            const bool out_f32 = (P.flags & kProbOutF32) != 0;
            const bool e_f32 = (P.flags & kProbEF32) != 0;
            const int row0 = ti.m0 + HM * static_cast<int>(rank) + q * 32;
            const int row = row0 + lane;
            const bool row_ok = row < P.M;
            const bool has_e = (beta != 0.0f) && (P.E[0] != nullptr);
            const bool e_lo = has_e && !e_f32 && (P.E[1] != nullptr);
            const bool lo_out = !out_f32 && P.out[1] != nullptr;
            const size_t row_base = static_cast<size_t>(row) * P.ld;
            const uint32_t t_row = tmem_base + acc * ACC_COLS + (static_cast<uint32_t>(q * 32) << 16);

            // v[32] = alpha * acc + beta * E of one row (lane), E as 4 x 8 bf16 per plane
            auto combine_bf16 = [&](const uint32_t (&r)[32], const uint4 (&eh)[4], const uint4 (&el)[4], float (&v)[32]) {
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    const uint32_t hw[4] = {eh[g].x, eh[g].y, eh[g].z, eh[g].w};
                    const uint32_t lw[4] = {el[g].x, el[g].y, el[g].z, el[g].w};
#pragma unroll
                    for (int h = 0; h < 4; ++h) {
                        const float e0 = bf16_lo_to_f32(hw[h]) + bf16_lo_to_f32(lw[h]);
                        const float e1 = bf16_hi_to_f32(hw[h]) + bf16_hi_to_f32(lw[h]);
                        v[8 * g + 2 * h] = fmaf(beta, e0, alpha * __uint_as_float(r[8 * g + 2 * h]));
                        v[8 * g + 2 * h + 1] = fmaf(beta, e1, alpha * __uint_as_float(r[8 * g + 2 * h + 1]));
                    }
                }
            };
            // Mirror store of a symmetric output, per lane: element (row, col) with col > row
            // also goes to (col, row); for a fixed col the 32 lanes write 32 consecutive rows.
            auto mirror_per_lane = [&](int col0, const float (&v)[32]) {
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int col = col0 + j;
                    if (row_ok && col > row && col < P.N) {
                        const size_t off = static_cast<size_t>(col) * P.ld + row;
                        if (out_f32) {
                            static_cast<float*>(P.out[0])[off] = v[j];
                        } else {
                            const __nv_bfloat16 hv = __float2bfloat16_rn(v[j]);
                            static_cast<__nv_bfloat16*>(P.out[0])[off] = hv;
                            if (lo_out)
                                static_cast<__nv_bfloat16*>(P.out[1])[off] = __float2bfloat16_rn(v[j] - __bfloat162float(hv));
                        }
                    }
                }
            };
            // Direct store of row `row` (per lane), upper triangle only for symmetric outputs.
            auto direct_per_lane = [&](int col0, float (&v)[32]) {
                if (!(row_ok && (!sym || col0 + 31 >= row))) return;
                if (out_f32) {
                    float* o = static_cast<float*>(P.out[0]) + row_base;
#pragma unroll
                    for (int g = 0; g < 8; ++g) {
                        const int cg = col0 + 4 * g;
                        if (cg >= P.N) continue;
                        if (!sym || cg >= row) {
                            *reinterpret_cast<float4*>(o + cg) = make_float4(v[4 * g], v[4 * g + 1], v[4 * g + 2], v[4 * g + 3]);
                        } else if (cg + 3 >= row) {
#pragma unroll
                            for (int j = 0; j < 4; ++j)
                                if (cg + j >= row) o[cg + j] = v[4 * g + j];
                        }
                    }
                } else {
                    __nv_bfloat16* o0 = static_cast<__nv_bfloat16*>(P.out[0]) + row_base;
                    __nv_bfloat16* o1 = static_cast<__nv_bfloat16*>(P.out[1]) + row_base;
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        const int cg = col0 + 8 * g;
                        if (cg >= P.N) continue;
                        float lo[8];
#pragma unroll
                        for (int j = 0; j < 8; ++j)
                            lo[j] = v[8 * g + j] - __bfloat162float(__float2bfloat16_rn(v[8 * g + j]));
                        if (!sym || cg >= row) {
                            store_bf16x8(o0 + cg, v + 8 * g);
                            if (lo_out) store_bf16x8(o1 + cg, lo);
                        } else if (cg + 7 >= row) {
#pragma unroll
                            for (int j = 0; j < 8; ++j) {
                                if (cg + j >= row) {
                                    o0[cg + j] = __float2bfloat16_rn(v[8 * g + j]);
                                    if (lo_out) o1[cg + j] = __float2bfloat16_rn(lo[j]);
                                }
                            }
                        }
                    }
                }
            };

            if (!out_f32 && !e_f32) {
                // ---------------- bf16 E and output: coalesced accesses through the staging buffers
                // Plane 0 of E for chunk c goes by cp.async (16 bytes per lane: rows crow + 8i,
                // segment cseg; zero-filled outside the matrix) into staging slot c & 1, one
                // commit group per chunk, so it is in flight while the previous chunk is processed.
                auto prefetch_e = [&](int c) {
                    const int col0 = ti.n0 + c * 32;
                    // chunks entirely below the diagonal of a symmetric output store nothing
                    if (has_e && col0 < P.N && !(sym && col0 + 31 < row0)) {
                        const __nv_bfloat16* e = static_cast<const __nv_bfloat16*>(P.E[0]);
                        uint8_t* dst = stg_e + (c & 1) * STG_BYTES;
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const int rr = row0 + crow + 8 * i;
                            const bool in = rr < P.M;
                            const __nv_bfloat16* src = in ? e + static_cast<size_t>(rr) * P.ld + col0 + 8 * cseg : e;
                            cp_async16_zfill(dst + stg_off64(crow + 8 * i, cseg), src, in ? 16 : 0);
                        }
                    }
                    cp_async_commit();
                };
                // a split E's plane 1 for chunk c, read directly (coalesced) and turned into rows
                auto load_e_lo = [&](int c, uint4 (&el)[4]) {
                    const int col0 = ti.n0 + c * 32;
                    const __nv_bfloat16* e = static_cast<const __nv_bfloat16*>(P.E[1]);
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int rr = row0 + crow + 8 * i;
                        el[i] = rr < P.M ? __ldg(reinterpret_cast<const uint4*>(e + static_cast<size_t>(rr) * P.ld + col0 + 8 * cseg))
                                         : make_uint4(0, 0, 0, 0);
                    }
#pragma unroll
                    for (int i = 0; i < 4; ++i) *reinterpret_cast<uint4*>(stg + stg_off64(crow + 8 * i, cseg)) = el[i];
                    __syncwarp();
#pragma unroll
                    for (int g = 0; g < 4; ++g) el[g] = *reinterpret_cast<const uint4*>(stg + stg_off64(lane, g));
                    __syncwarp();
                };
                prefetch_e(c_beg);
                // the chunk loop synchronises the warp: every lane takes the same decision
                if (!__all_sync(0xffffffffu, mbar_wait(&tfull_bar[acc], acc_phase, abort_flag, dev_status))) {
                    cp_async_wait_all();
                    break;
                }
                tc_fence_after();
#pragma unroll 1
                for (int c = c_beg; c < c_end; ++c) {
                    const int col0 = ti.n0 + c * 32;
                    if (col0 >= P.N) break;  // uniform across the warp
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(t_row + c * 32, r);
                    if (c + 1 < c_end) prefetch_e(c + 1);
                    else cp_async_commit();
                    tmem_ld_wait();
                    // the chunk against the diagonal (uniform): rows row0 .. row0 + 31, columns
                    // col0 .. col0 + 31, both multiples of 32
                    const bool below = sym && col0 < row0;
                    const bool diag = sym && col0 == row0;
                    uint4 eh[4], el[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) { eh[i] = make_uint4(0, 0, 0, 0); el[i] = make_uint4(0, 0, 0, 0); }
                    cp_async_wait_group<1>();   // this lane's copies of chunk c have landed
                    __syncwarp();               // ... and every lane's
                    if (has_e && !below) {
                        const uint8_t* src = stg_e + (c & 1) * STG_BYTES;
#pragma unroll
                        for (int g = 0; g < 4; ++g) eh[g] = *reinterpret_cast<const uint4*>(src + stg_off64(lane, g));
                        if (e_lo) load_e_lo(c, el);
                    }
                    __syncwarp();               // slot c & 1 is free for chunk c + 2
                    float v[32];
                    combine_bf16(r, eh, el, v);
                    if (diag) {
                        direct_per_lane(col0, v);
                        mirror_per_lane(col0, v);
                    } else if (!below) {
                        // direct store (hi, then lo): per-lane rows -> staging -> 8 rows x 64 B
                        // per instruction.  N is a multiple of 8: a 16-byte segment is wholly
                        // inside or outside the matrix.
#pragma unroll 1
                        for (int pl = 0; pl < (lo_out ? 2 : 1); ++pl) {
#pragma unroll
                            for (int g = 0; g < 4; ++g) {
                                float w[8];
#pragma unroll
                                for (int j = 0; j < 8; ++j) {
                                    const float x = v[8 * g + j];
                                    w[j] = pl == 0 ? x : x - __bfloat162float(__float2bfloat16_rn(x));
                                }
                                uint4 pk;
                                pk.x = pack_bf16x2(w[0], w[1]); pk.y = pack_bf16x2(w[2], w[3]);
                                pk.z = pack_bf16x2(w[4], w[5]); pk.w = pack_bf16x2(w[6], w[7]);
                                *reinterpret_cast<uint4*>(stg + stg_off64(lane, g)) = pk;
                            }
                            __syncwarp();
                            __nv_bfloat16* o = static_cast<__nv_bfloat16*>(P.out[pl]);
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                const int rr = row0 + crow + 8 * i;
                                const int cc = col0 + 8 * cseg;
                                const uint4 val = *reinterpret_cast<const uint4*>(stg + stg_off64(crow + 8 * i, cseg));
                                if (rr < P.M && cc < P.N)
                                    *reinterpret_cast<uint4*>(o + static_cast<size_t>(rr) * P.ld + cc) = val;
                            }
                            if (sym) {
                                // mirror: the staged plane transposed into stg_t, which then
                                // leaves as 8 rows x 64 B per instruction
                                stg_transpose32(stg, stg_t, lane);
                                __syncwarp();
#pragma unroll
                                for (int i = 0; i < 4; ++i) {
                                    const int rr = col0 + crow + 8 * i;     // mirrored row
                                    const int cc = row0 + 8 * cseg;         // mirrored columns
                                    const uint4 val = *reinterpret_cast<const uint4*>(stg_t + stg_off64(crow + 8 * i, cseg));
                                    if (rr < P.N && cc < P.M)
                                        *reinterpret_cast<uint4*>(o + static_cast<size_t>(rr) * P.ld + cc) = val;
                                }
                            }
                            __syncwarp();
                        }
                    }
                }
                cp_async_wait_all();   // the trailing (empty) groups: nothing is left in flight
            } else {
                // ---------------- fp32 E or output: per-lane rows
                // E of chunk c for this row: bf16 -> ew[0..3] plane 0, ew[4..7] plane 1; fp32 -> ew[0..7]
                auto load_e = [&](int c, uint4 (&ew)[8]) {
                    const int col0 = ti.n0 + c * 32;
                    const bool need = has_e && row_ok && col0 < P.N && (!sym || col0 + 31 >= row);
#pragma unroll
                    for (int g = 0; g < 8; ++g) ew[g] = make_uint4(0, 0, 0, 0);
                    if (!need) return;
                    if (e_f32) {
                        const float* e0 = static_cast<const float*>(P.E[0]) + row_base + col0;
#pragma unroll
                        for (int g = 0; g < 8; ++g)
                            if (col0 + 4 * g < P.N) ew[g] = __ldg(reinterpret_cast<const uint4*>(e0 + 4 * g));
                    } else {
                        const __nv_bfloat16* e0 = static_cast<const __nv_bfloat16*>(P.E[0]) + row_base + col0;
                        const __nv_bfloat16* e1 = static_cast<const __nv_bfloat16*>(P.E[1]) + row_base + col0;
#pragma unroll
                        for (int g = 0; g < 4; ++g) {
                            if (col0 + 8 * g < P.N) {
                                ew[g] = __ldg(reinterpret_cast<const uint4*>(e0 + 8 * g));
                                if (e_lo) ew[4 + g] = __ldg(reinterpret_cast<const uint4*>(e1 + 8 * g));
                            }
                        }
                    }
                };
                uint4 ew[8];
                load_e(c_beg, ew);
                if (!__all_sync(0xffffffffu, mbar_wait(&tfull_bar[acc], acc_phase, abort_flag, dev_status))) break;
                tc_fence_after();
#pragma unroll 1
                for (int c = c_beg; c < c_end; ++c) {
                    const int col0 = ti.n0 + c * 32;
                    if (col0 >= P.N) break;  // uniform across the warp
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(t_row + c * 32, r);
                    uint4 nw[8];
                    if (c + 1 < c_end) load_e(c + 1, nw);
                    tmem_ld_wait();
                    float v[32];
                    if (e_f32) {
#pragma unroll
                        for (int g = 0; g < 8; ++g) {
                            const uint32_t w4[4] = {ew[g].x, ew[g].y, ew[g].z, ew[g].w};
#pragma unroll
                            for (int h = 0; h < 4; ++h)
                                v[4 * g + h] = fmaf(beta, __uint_as_float(w4[h]), alpha * __uint_as_float(r[4 * g + h]));
                        }
                    } else {
                        const uint4 eh[4] = {ew[0], ew[1], ew[2], ew[3]};
                        const uint4 el[4] = {ew[4], ew[5], ew[6], ew[7]};
                        combine_bf16(r, eh, el, v);
                    }
                    direct_per_lane(col0, v);
                    if (sym) mirror_per_lane(col0, v);
#pragma unroll
                    for (int g = 0; g < 8; ++g) ew[g] = nw[g];
                }
            }
            tc_fence_before();
            mbar_arrive_cluster(tempty_leader + acc * 8u);
            if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
        }
    }
    tc_fence_before();
    cluster_sync();     // no CTA leaves while its pair may still touch its memory
    tc_fence_after();
    if (warp == 2) tmem_dealloc_pair(tmem_base, TMEM_COLS);
}

}  // namespace

size_t tc_gemm_smem_bytes() { return SMEM_TOTAL; }

cudaError_t tc_gemm_launch(const TcProblem* d_probs, const uint32_t* d_tiles, int num_tiles, unsigned* d_status,
                           int num_sms, cudaStream_t stream) {
    if (num_tiles <= 0) return cudaSuccess;
    // Function attributes and the cluster occupancy are per device: set up once on each.
    // (Launches run under the plan cache's lock, so this needs none of its own.)
    constexpr int kMaxDevices = 64;
    static int max_pairs_of[kMaxDevices] = {};
    int dev = 0;
    cudaError_t de = cudaGetDevice(&dev);
    if (de != cudaSuccess) return de;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    int& max_pairs = max_pairs_of[dev];
    if (max_pairs == 0) {
        cudaError_t e = cudaFuncSetAttribute(tc_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_TOTAL);
        if (e != cudaSuccess) return e;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2 * (num_sms / 2), 1, 1);
        cfg.blockDim = dim3(kTcThreads, 1, 1);
        cfg.dynamicSmemBytes = SMEM_TOTAL;
        cudaLaunchAttribute attr;
        attr.id = cudaLaunchAttributeClusterDimension;
        attr.val.clusterDim.x = 2;
        attr.val.clusterDim.y = 1;
        attr.val.clusterDim.z = 1;
        cfg.attrs = &attr;
        cfg.numAttrs = 1;
        int clusters = 0;
        e = cudaOccupancyMaxActiveClusters(&clusters, tc_gemm_kernel, &cfg);
        if (e != cudaSuccess || clusters <= 0) {
            cudaGetLastError();   // fall back to one pair per two SMs; leave no error pending
            clusters = num_sms / 2;
        }
        max_pairs = clusters;
    }
    const int pairs = num_tiles < max_pairs ? num_tiles : max_pairs;
    // The grid is at most the resident capacity (every CTA runs from the start), so CTAs of the
    // next launch that wait on this grid only take SMs that finished CTAs released.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * pairs, 1, 1);
    cfg.blockDim = dim3(kTcThreads, 1, 1);
    cfg.dynamicSmemBytes = SMEM_TOTAL;
    cfg.stream = stream;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, tc_gemm_kernel, d_probs, d_tiles, num_tiles, d_status);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace muon
