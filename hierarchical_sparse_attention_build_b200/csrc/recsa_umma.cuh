// Pooler product on the 5th-generation tensor cores (tcgen05, accumulator in TMEM).
//
// key = W @ mean for up to 128 nodes at once: D[m][o] = sum_k A[m][k] * B[o][k] with
// A = the nodes' fp32 key means and B = W (row-major [o][k], i.e. K-major), or with the
// roles exchanged (A = W, B = the means, D[o][m]) where few nodes need a product: an MMA
// instruction costs about the same at N = 16 as at N = 128, 2.5K against 3.3K cycles for the
// 48 of a product, so a short N helps only a little, and both forms give each element
// the same fp32 result (checked element by element on B200, and by the append-equals-build
// tests).  A single
// bf16 pass would round the operands to 8 bits, well above the precision of a stored bf16
// row, so each fp32 operand is split exactly into three bf16 parts x = x0 + x1 + x2
// (x0 = bf16(x), x1 = bf16(x - x0), x2 = bf16(x - x0 - x1)) and the six products whose
// terms reach 2^-16 of the result are accumulated in fp32: the dropped ones (x1*y2, x2*y1,
// x2*y2) are below 2^-24 relative.  Every caller issues the same products in the same order
// into a zeroed accumulator, so a node's key does not depend on which kernel built it or on
// the other rows of its tile.
#pragma once

#include <cstdint>

#include "recsa_device.cuh"

namespace recsa {
namespace umma {

constexpr int kM = 128;              // accumulator rows (nodes)
constexpr int kN = 128;              // outputs
constexpr int kParts = 3;            // bf16 parts of an fp32 operand
constexpr int kPartBytes = kM * kD * 2;  // one bf16 part of a 128 x 128 operand: 32 KB
constexpr int kOperandBytes = kParts * kPartBytes;
constexpr uint32_t kTmemCols = 128;  // one fp32 accumulator of 128 x 128

// Byte offset of element (r, k) of a K-major operand without swizzle: 8 x 8 core matrices
// of 128 bytes (row r % 8 at 16 r % 8, 8 consecutive k in a row), 16 core matrices along K
// per group of 8 rows (the leading-dimension step, LBO = 128 bytes), row groups 2048 bytes
// apart (the stride-dimension step, SBO).
__host__ __device__ constexpr int operand_offset(int r, int k) {
  return ((r >> 3) * 16 + (k >> 3)) * 128 + (r & 7) * 16 + (k & 7) * 2;
}
constexpr uint32_t kLBO = 128, kSBO = 2048;

// Shared-memory matrix descriptor: start address, LBO and SBO in 16-byte units, descriptor
// version 1, no swizzle.
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3fffu) | ((uint64_t)(kLBO >> 4) << 16) | ((uint64_t)(kSBO >> 4) << 32) |
         (1ull << 46);
}
// Instruction descriptor of kind::f16: fp32 accumulator, bf16 A and B, both K-major, M = 128,
// N = n (a multiple of 16 up to 256).
__host__ __device__ constexpr uint32_t idesc_n(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(kM >> 4) << 24);
}
constexpr uint32_t kIdesc = idesc_n(kN);

// the six products (A part, B part), smallest terms first
__host__ __device__ constexpr int prod_a(int i) { return i == 0 ? 1 : i == 1 ? 2 : i == 2 ? 0 : i == 3 ? 1 : i == 4 ? 0 : 0; }
__host__ __device__ constexpr int prod_b(int i) { return i == 0 ? 1 : i == 1 ? 0 : i == 2 ? 2 : i == 3 ? 0 : i == 4 ? 1 : 0; }
constexpr int kProducts = 6;

// x = p0 + p1 + p2 in bf16 parts (round to nearest even at each step; the residues are exact in fp32)
__device__ __forceinline__ void split3(float x, uint32_t &p0, uint32_t &p1, uint32_t &p2) {
  p0 = f32_to_bf16_bits(x);
  const float r1 = x - __uint_as_float(p0 << 16);
  p1 = f32_to_bf16_bits(r1);
  const float r2 = r1 - __uint_as_float(p1 << 16);
  p2 = f32_to_bf16_bits(r2);
}

// Four consecutive k (k % 4 == 0) of row r, as the three parts, into the operand at `base`.
__device__ __forceinline__ void store_row4_parts(unsigned char *base, int r, int k, const float x[4]) {
  uint32_t p[3][4];
#pragma unroll
  for (int i = 0; i < 4; ++i) split3(x[i], p[0][i], p[1][i], p[2][i]);
#pragma unroll
  for (int q = 0; q < kParts; ++q)
    *reinterpret_cast<uint2 *>(base + q * kPartBytes + operand_offset(r, k)) =
        make_uint2(p[q][0] | (p[q][1] << 16), p[q][2] | (p[q][3] << 16));
}

__device__ __forceinline__ void tmem_alloc(uint32_t *dst, uint32_t ncols) {  // one whole warp
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {  // one whole warp
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {  // one whole warp
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void fence_before_sync() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after_sync() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
// generic-proxy writes to shared memory become visible to the tensor cores' reads
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ void mma(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                    uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\ttcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(
          tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// arrives on the mbarrier once every MMA issued before it by this thread has completed
__device__ __forceinline__ void commit(uint64_t *bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// One thread: D = A @ B^T over K = 128 as the six split products (A, B: operands at
// shared addresses a_s, b_s, each three parts of kPartBytes).
__device__ __forceinline__ void issue_pooler(uint32_t tmem_d, uint32_t a_s, uint32_t b_s) {
  uint32_t acc = 0;
#pragma unroll
  for (int pi = 0; pi < kProducts; ++pi) {
    const uint32_t a0 = a_s + prod_a(pi) * kPartBytes, b0 = b_s + prod_b(pi) * kPartBytes;
#pragma unroll
    for (int ks = 0; ks < kD / 16; ++ks) {  // 16 k per instruction: two core matrices along K
      mma(tmem_d, smem_desc(a0 + ks * 256), smem_desc(b0 + ks * 256), kIdesc, acc);
      acc = 1;
    }
  }
}

// One thread: the same six products in the same order with the operands' roles exchanged,
// D[o][m] = sum_k W[o][k] * mean[m][k] for nodes m < n (n a multiple of 16): W's parts at
// w_s (rows o), the means' parts at m_s (rows m).
__device__ __forceinline__ void issue_pooler_t(uint32_t tmem_d, uint32_t w_s, uint32_t m_s, int n) {
  const uint32_t idesc = idesc_n(n);
  uint32_t acc = 0;
#pragma unroll
  for (int pi = 0; pi < kProducts; ++pi) {
    const uint32_t w0 = w_s + prod_b(pi) * kPartBytes, m0 = m_s + prod_a(pi) * kPartBytes;
#pragma unroll
    for (int ks = 0; ks < kD / 16; ++ks) {
      mma(tmem_d, smem_desc(w0 + ks * 256), smem_desc(m0 + ks * 256), idesc, acc);
      acc = 1;
    }
  }
}

// 32 consecutive fp32 columns of the accumulator lane this thread reads (warp w reads lanes
// 32 (w % 4) .. 32 (w % 4) + 31), after which tcgen05.wait::ld must run before use.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]),
        "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]),
        "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]),
        "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// W into an operand (three parts): element (o, k) = W[o][k].  A warp's 32 pieces of 4 k
// cover rows 8g .. 8g+7 and k 16c .. 16c+15: two whole core matrices, so each 8-byte store
// fills 256 contiguous bytes without a bank conflict (a row's pieces are 128 bytes apart).
template <int NT, int kMaxBatch = 4>
__device__ __forceinline__ void load_pooler_operand(const float *__restrict__ W, unsigned char *b_ops, int tid) {
  constexpr int kPer = kD * kD / 4 / NT;  // pieces a thread
  constexpr int kBatch = kPer < kMaxBatch ? kPer : kMaxBatch;  // loads in flight at once
  static_assert(kPer * NT == kD * kD / 4 && kPer % kBatch == 0, "the thread count divides the pooler's pieces");
#pragma unroll 1
  for (int i0 = 0; i0 < kPer; i0 += kBatch) {
    float4 w[kBatch];
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      const int e = tid + (i0 + i) * NT, c = e >> 5, lane = e & 31;
      const int o = (c & 15) * 8 + (lane & 7), k = (c >> 4) * 16 + (lane >> 3) * 4;
      w[i] = __ldg(reinterpret_cast<const float4 *>(W + o * kD + k));
    }
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      const int e = tid + (i0 + i) * NT, c = e >> 5, lane = e & 31;
      const int o = (c & 15) * 8 + (lane & 7), k = (c >> 4) * 16 + (lane >> 3) * 4;
      const float x[4] = {w[i].x, w[i].y, w[i].z, w[i].w};
      store_row4_parts(b_ops, o, k, x);
    }
  }
}

}  // namespace umma
}  // namespace recsa
