// Stage 1 of MuSe for DIPOLE summaries on the fifth-generation tensor cores
// (tcgen05, TMEM), bf16 inputs.
//
// For key cluster j of a key block and every query cluster i of the paired
// query block, the dipole-corrected summary value is
//   u_ij = (1/n_j) sum_{t in j} v_t (1 + s nu_i . (k_t - mu_j))
// (newx.sg page "Multipole Semantic Attention: A Fast Approximation of Softmax
// Attention for Pretraining", Abstract: monopole plus dipole corrections; the
// first-order term of the kept cross term, gist.science page, Technical
// Summary, Core Mechanisms, residual decomposition).  One CTA of 128 threads
// per (query problem, key cluster), members in chunks of 128 rows:
//   G = K nu^T      tcgen05.mma kind::f16, M=128 members, N=128 query
//                   clusters, bf16 keys x bf16 hi + lo split of nu (two MMAs
//                   into one fp32 TMEM accumulator);
//   W = 1 + s (G - nu . mu_j)   thread t forms member t's row as an fp16
//                   hi + lo pair and stores both as MN-major A operands;
//   U += W_hi^T V + W_lo^T V   tcgen05.mma, M=128 query clusters, N=D,
//                   K=128 members, fp16 operands (both MN-major: rows as they
//                   are formed or stored), fp32 accumulator resident in TMEM
//                   over the chunks.  The split keeps u_ij accurate when the
//                   dipole factors are large (heavy-tailed keys): one fp16
//                   rounding of W costs 2^-11 |W| per member.
// Thread i then writes u_ij = U[i] / n_j as an fp16 hi + lo pair (128
// contiguous bytes per 64 dimensions each), the operand form of stage 2.
#include <cuda_fp16.h>
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace muse {

namespace {

constexpr int kR = 128;  // rows per operand tile: members, query clusters
constexpr int kS1T = 128;

__device__ inline uint32_t s32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ inline uint32_t swz(int r, int q) { return r * 128 + ((q ^ (r & 7)) << 4); }
__device__ inline uint64_t desc_k(uint32_t a) {
  return (uint64_t)((a >> 4) & 0x3FFF) | (1ull << 16) | ((uint64_t)(1024 >> 4) << 32) |
         (1ull << 46) | (2ull << 61);
}
__device__ inline uint64_t desc_mn(uint32_t a, uint32_t lbo) {
  return (uint64_t)((a >> 4) & 0x3FFF) | ((uint64_t)((lbo >> 4) & 0x3FFF) << 16) |
         ((uint64_t)(1024 >> 4) << 32) | (1ull << 46) | (2ull << 61);
}
__device__ inline void umma(uint32_t tmem, uint64_t ad, uint64_t bd, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tmem),
      "l"(ad), "l"(bd), "r"(idesc), "r"(acc));
}
__device__ inline void umma_commit(uint32_t mbar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(mbar)
               : "memory");
}
__device__ inline bool wait_mbar(uint32_t mbar, uint32_t parity) {
  for (int it = 0; it < (1 << 20); ++it) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(done)
        : "r"(mbar), "r"(parity)
        : "memory");
    if (done) return true;
  }
  return false;
}
__device__ inline void tld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ inline void tld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory"); }
// The wait, tied to the 64 registers of four loads so that no use of them
// moves above it.
__device__ inline void tld_wait4(uint32_t (&r)[4][16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;\n"
               : "+r"(r[0][0]), "+r"(r[0][1]), "+r"(r[0][2]), "+r"(r[0][3]), "+r"(r[0][4]), "+r"(r[0][5]),
                 "+r"(r[0][6]), "+r"(r[0][7]), "+r"(r[0][8]), "+r"(r[0][9]), "+r"(r[0][10]),
                 "+r"(r[0][11]), "+r"(r[0][12]), "+r"(r[0][13]), "+r"(r[0][14]), "+r"(r[0][15]),
                 "+r"(r[1][0]), "+r"(r[1][1]), "+r"(r[1][2]), "+r"(r[1][3]), "+r"(r[1][4]), "+r"(r[1][5]),
                 "+r"(r[1][6]), "+r"(r[1][7]), "+r"(r[1][8]), "+r"(r[1][9]), "+r"(r[1][10]),
                 "+r"(r[1][11]), "+r"(r[1][12]), "+r"(r[1][13]), "+r"(r[1][14]), "+r"(r[1][15])
               :
               : "memory");
  asm volatile(""
               : "+r"(r[2][0]), "+r"(r[2][1]), "+r"(r[2][2]), "+r"(r[2][3]), "+r"(r[2][4]), "+r"(r[2][5]),
                 "+r"(r[2][6]), "+r"(r[2][7]), "+r"(r[2][8]), "+r"(r[2][9]), "+r"(r[2][10]),
                 "+r"(r[2][11]), "+r"(r[2][12]), "+r"(r[2][13]), "+r"(r[2][14]), "+r"(r[2][15]),
                 "+r"(r[3][0]), "+r"(r[3][1]), "+r"(r[3][2]), "+r"(r[3][3]), "+r"(r[3][4]), "+r"(r[3][5]),
                 "+r"(r[3][6]), "+r"(r[3][7]), "+r"(r[3][8]), "+r"(r[3][9]), "+r"(r[3][10]),
                 "+r"(r[3][11]), "+r"(r[3][12]), "+r"(r[3][13]), "+r"(r[3][14]), "+r"(r[3][15])
               :
               : "memory");
}
__device__ inline void fence_before() { asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory"); }
__device__ inline void fence_after() { asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory"); }
__device__ inline void fence_async() { asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory"); }
__device__ inline void cp16(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src),
               "r"(src_bytes));
}
__device__ inline void cp_commit_wait() {
  asm volatile("cp.async.commit_group;\ncp.async.wait_group 0;\n" ::: "memory");
}
__device__ inline uint32_t h2bits(float x, float y) {
  const __half2 h = __floats2half2_rn(x, y);
  return *reinterpret_cast<const uint32_t*>(&h);
}
// fp16 pair (x, y) = hi + lo (residual 2^-22 relative).
__device__ inline void split_h2bits(float x, float y, uint32_t& hi, uint32_t& lo) {
  const __half2 h = __floats2half2_rn(x, y);
  const float2 f = __half22float2(h);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = h2bits(x - f.x, y - f.y);
}

template <int D>
struct S1Layout {
  static constexpr int KB = D / 64;
  static constexpr int OP = KB * kR * 128;  // one [128 rows][D] 16-bit operand, bytes
  static constexpr int NH = 0;              // nu hi, K-major
  static constexpr int NL = NH + OP;        // nu lo
  static constexpr int KM = NL + OP;        // member keys, K-major
  static constexpr int VM = KM + OP;        // member values (fp16), MN-major B
  static constexpr int W = VM + OP;         // [2 cluster chunks][128 members][128 B], MN-major A
  // fp16 residual of W, same layout: it takes the nu operands' place (2 x
  // 128 x 128 bytes fit in NH, or in NH and NL for D = 64), which the G MMA
  // of the member chunk has finished with; every chunk reloads nu
  static constexpr int WL = NH;
  static constexpr int NM = W + 2 * kR * 128;  // nu_i . mu_j
  static constexpr int MU = NM + kR * 4;
  static constexpr int TOTAL = MU + D * 4 + 1024;
};

}  // namespace

template <int D>
__global__ void __launch_bounds__(kS1T) stage1_dipole_tc_kernel(AttnArgs a, Stage1 s1, int qp0) {
  using Lt = S1Layout<D>;
  constexpr int KB = Lt::KB;
  extern __shared__ __align__(1024) unsigned char s1_raw[];
  unsigned char* sm = s1_raw + ((1024 - (s32(s1_raw) & 1023)) & 1023);
  float* nm = reinterpret_cast<float*>(sm + Lt::NM);
  float* mu = reinterpret_cast<float*>(sm + Lt::MU);
  __shared__ __align__(8) uint64_t mbar[2];  // G ready, U step done
  __shared__ uint32_t tslot;

  const int lq = blockIdx.x, qpid = qp0 + lq, j = blockIdx.y;
  const Prob pq = prob_of(a.qg, qpid);
  if ((a.dense_lv >> pq.level) & 1) return;  // that level's far field runs per key token
  const int kpid = kv_problem(a, qpid);
  const Prob pk = prob_of(a.kg, kpid);
  if (j >= pk.C) return;
  const int tid = threadIdx.x, warp = tid >> 5;
  const int Cq = a.Cq, Ck = a.Ck;
  const int nj = a.ks.counts[(size_t)kpid * Ck + j];
  const size_t ij0 = ((size_t)lq * Cq) * Ck + j;  // + i * Ck
  if (nj == 0) {
    for (int i = tid; i < pq.C; i += kS1T) {
      s1.logW[ij0 + (size_t)i * Ck] = -INFINITY;
      s1.fbias[ij0 + (size_t)i * Ck] = -INFINITY;
    }
    return;
  }
  const float lognj = logf((float)nj);
  for (int i = tid; i < pq.C; i += kS1T) {
    s1.logW[ij0 + (size_t)i * Ck] = lognj;
    s1.fbias[ij0 + (size_t)i * Ck] = lognj;
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(
                     s32(&tslot)),
                 "r"(256));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n");
  }
  if (tid == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;\n" ::"r"(s32(&mbar[0])));
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;\n" ::"r"(s32(&mbar[1])));
    asm volatile("fence.mbarrier_init.release.cluster;\n");
  }
  const float* mug = a.ks.cent32 + ((size_t)kpid * Ck + j) * D;
  for (int d = tid; d < D; d += kS1T) mu[d] = mug[d];
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tbase = tslot;
  const uint32_t tl = tbase + ((uint32_t)(warp * 32) << 16);  // this warp's lanes
  const uint32_t tG = tbase, tU = tbase + kR;
  const int off = a.ks.off[(size_t)kpid * (Ck + 1) + j];
  const int* perm = a.ks.perm + pk.slot0;
  const __nv_bfloat16* Kx = static_cast<const __nv_bfloat16*>(a.kg.X);
  const float s = a.scale;
  const float inv_n = 1.f / (float)nj;
  const uint32_t sb = s32(sm);
  // G: f32 accumulator, bf16 A (members) and B (query clusters), both K-major
  const uint32_t id_g = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kR >> 3) << 17) |
                        ((uint32_t)(kR >> 4) << 24);
  // U: f32 accumulator, f16 A = W^T and B = V, both MN-major, N = D
  const uint32_t id_u = (1u << 4) | (1u << 15) | (1u << 16) | ((uint32_t)(D >> 3) << 17) |
                        ((uint32_t)(kR >> 4) << 24);
  uint32_t ph[2] = {0u, 0u};
  bool ok = true;

  // members of this CTA's rows in the member-row loads below: thread t copies
  // the 16-byte pieces t, t + 128, ... of the 128 x KB x 8 grid, rows
  // (t + 128 m) / (KB 8)
  constexpr int kPieces = kR * KB * 8 / kS1T;
  for (int i0 = 0; i0 < pq.C; i0 += kR) {
    const int ic = imin(kR, pq.C - i0);
    for (int t0 = 0; t0 < nj; t0 += kR) {
      const int nt = imin(kR, nj - t0);
      // the copies first (query centroids as the bf16 split, rows past ic
      // zero; member keys and values through the permutation, rows past nt
      // zero); the dot products nu_i . mu_j run while they are in flight
      for (int e = tid; e < kR * KB * 8; e += kS1T) {
        const int r = e / (KB * 8), q = e - r * (KB * 8), kb = q >> 3, c = q & 7;
        const bool live = r < ic;
        const size_t o = ((size_t)qpid * Cq + i0 + (live ? r : 0)) * D + kb * 64 + c * 8;
        const uint32_t so = kb * kR * 128 + swz(r, c);
        cp16(sb + Lt::NH + so, a.qs.cbf_hi + o, live ? 16 : 0);
        cp16(sb + Lt::NL + so, a.qs.cbf_lo + o, live ? 16 : 0);
      }
      {
        int rows[kPieces];  // every permutation entry read before the first copy
#pragma unroll
        for (int m = 0; m < kPieces; ++m) {
          const int r = (tid + m * kS1T) / (KB * 8);
          rows[m] = r < nt ? perm[off + t0 + r] : -1;
        }
#pragma unroll
        for (int m = 0; m < kPieces; ++m) {
          const int e = tid + m * kS1T;
          const int r = e / (KB * 8), q = e - r * (KB * 8), kb = q >> 3, c = q & 7;
          const long long row = pk.row0 + (rows[m] >= 0 ? rows[m] : 0);
          const uint32_t so = kb * kR * 128 + swz(r, c);
          cp16(sb + Lt::KM + so, Kx + row * D + kb * 64 + c * 8, rows[m] >= 0 ? 16 : 0);
          cp16(sb + Lt::VM + so, a.V16 + row * D + kb * 64 + c * 8, rows[m] >= 0 ? 16 : 0);
        }
      }
      if (t0 == 0) {  // nu_i . mu_j of this pass: every load in flight at once
        float dt = 0.f;
        if (tid < ic) {
          const float4* nu = reinterpret_cast<const float4*>(a.qs.cent32 + ((size_t)qpid * Cq + i0 + tid) * D);
          float4 v[D / 4];
#pragma unroll
          for (int d4 = 0; d4 < D / 4; ++d4) v[d4] = nu[d4];
#pragma unroll
          for (int d4 = 0; d4 < D / 4; ++d4) {
            dt = fmaf(v[d4].x, mu[4 * d4], dt);
            dt = fmaf(v[d4].y, mu[4 * d4 + 1], dt);
            dt = fmaf(v[d4].z, mu[4 * d4 + 2], dt);
            dt = fmaf(v[d4].w, mu[4 * d4 + 3], dt);
          }
        }
        nm[tid] = dt;
      }
      cp_commit_wait();
      fence_async();
      fence_before();
      __syncthreads();
      fence_after();
      if (tid == 0) {
        for (int kb = 0; kb < KB; ++kb) {
          const uint64_t ad = desc_k(sb + Lt::KM + kb * kR * 128);
          const uint64_t hd = desc_k(sb + Lt::NH + kb * kR * 128);
          const uint64_t ld = desc_k(sb + Lt::NL + kb * kR * 128);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            umma(tG, ad + 2 * k, hd + 2 * k, id_g, (kb | k) ? 1u : 0u);
            umma(tG, ad + 2 * k, ld + 2 * k, id_g, 1u);
          }
        }
        umma_commit(s32(&mbar[0]));
      }
      ok = wait_mbar(s32(&mbar[0]), ph[0]) && ok;
      ph[0] ^= 1u;
      fence_after();
      // W row of member t = tid over the 128 query clusters; members past nt
      // get 0 so they add nothing
      // (the second half's TMEM loads run during the first half's arithmetic)
      uint32_t gall[2][4][16];
#pragma unroll
      for (int q = 0; q < 4; ++q) tld16(tl + 16 * q, gall[0][q]);
      tld_wait4(gall[0]);
#pragma unroll
      for (int q = 0; q < 4; ++q) tld16(tl + 64 + 16 * q, gall[1][q]);
#pragma unroll
      for (int h = 0; h < 2; ++h) {  // 64 query clusters per 128-byte row chunk
        if (h == 1) tld_wait4(gall[1]);
        uint32_t (&g4)[4][16] = gall[h];
        unsigned char* wrow = sm + Lt::W + h * kR * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          float w[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int ii = 8 * c + u;
            const float gv = __uint_as_float(g4[ii >> 4][ii & 15]);
            w[u] = tid < nt ? fmaf(s, gv - nm[64 * h + ii], 1.f) : 0.f;
          }
          uint32_t hi[4], lo[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) split_h2bits(w[2 * u], w[2 * u + 1], hi[u], lo[u]);
          *reinterpret_cast<uint4*>(wrow + swz(tid, c)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
          *reinterpret_cast<uint4*>(wrow + (Lt::WL - Lt::W) + swz(tid, c)) =
              make_uint4(lo[0], lo[1], lo[2], lo[3]);
        }
      }
      fence_async();
      fence_before();
      __syncthreads();
      fence_after();
      if (tid == 0) {
#pragma unroll
        for (int k = 0; k < kR / 16; ++k) {  // 16 members per step: two 8-row groups
          const uint64_t vd = desc_mn(sb + Lt::VM + 2048 * k, kR * 128);
          umma(tU, desc_mn(sb + Lt::W + 2048 * k, kR * 128), vd, id_u, (t0 > 0 || k > 0) ? 1u : 0u);
          umma(tU, desc_mn(sb + Lt::WL + 2048 * k, kR * 128), vd, id_u, 1u);
        }
        umma_commit(s32(&mbar[1]));
      }
      ok = wait_mbar(s32(&mbar[1]), ph[1]) && ok;  // the operands are reloaded next chunk
      ph[1] ^= 1u;
      fence_after();
    }
    // ---- u_ij = U[i] / n_j as fp16 hi + lo, thread i = query cluster i0 + i ---
#pragma unroll
    for (int d0 = 0; d0 < D; d0 += 16) {
      uint32_t r1[16];
      tld16(tl + kR + d0, r1);
      tld_wait();
      if (tid < ic) {
        const size_t o = (ij0 + (size_t)(i0 + tid) * Ck) * D + d0;
        uint32_t hi[8], lo[8];
#pragma unroll
        for (int u = 0; u < 8; ++u)
          split_h2bits(__uint_as_float(r1[2 * u]) * inv_n, __uint_as_float(r1[2 * u + 1]) * inv_n,
                       hi[u], lo[u]);
        reinterpret_cast<uint4*>(s1.Uh + o)[0] = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        reinterpret_cast<uint4*>(s1.Uh + o)[1] = make_uint4(hi[4], hi[5], hi[6], hi[7]);
        reinterpret_cast<uint4*>(s1.Ul + o)[0] = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        reinterpret_cast<uint4*>(s1.Ul + o)[1] = make_uint4(lo[4], lo[5], lo[6], lo[7]);
      }
    }
    fence_before();
    __syncthreads();  // the next pass overwrites the operands and G
    fence_after();
  }
  if (!ok && tid == 0) atomicOr(a.qs.err, kErrMmaWait);
  fence_before();
  __syncthreads();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tbase), "r"(256));
}

template <int D>
static void launch_s1tc(const AttnArgs& a, const Stage1& s1, int qp0, int nqp, cudaStream_t st) {
  // set on every launch: the attribute is per device, and the call is cheap
  cudaFuncSetAttribute(stage1_dipole_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       S1Layout<D>::TOTAL);
  stage1_dipole_tc_kernel<D><<<dim3(nqp, a.Ck), kS1T, S1Layout<D>::TOTAL, st>>>(a, s1, qp0);
}

void run_stage1_dipole_tc(const AttnArgs& a, const Stage1& s1, int qp0, int nqp, cudaStream_t st) {
  if (a.qg.D == 64)
    launch_s1tc<64>(a, s1, qp0, nqp, st);
  else
    launch_s1tc<128>(a, s1, qp0, nqp, st);
}

}  // namespace muse
