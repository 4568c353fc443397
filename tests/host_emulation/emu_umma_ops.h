// Host versions of the tcgen05 helpers of recsa_umma.cuh (test infrastructure).  TMEM is a
// per-CTA array of 128 lanes x 512 fp32 columns; an MMA reads its operands through the
// shared-memory descriptors it is given (start address, LBO, SBO of the no-swizzle K-major
// layout) and its shape through the instruction descriptor, and accumulates in fp32, k in
// order; the commit arrives on the mbarrier at once (the product is already done).
#pragma once
namespace emu {
extern thread_local float *t_tmem;  // [128][512] of the running CTA
}
namespace recsa {
namespace umma {
inline void tmem_alloc(uint32_t *dst, uint32_t) {
  if ((emu::t_tid & 31) == 0) *dst = 0u;  // lane 0, column 0
  __syncwarp();
}
inline void tmem_relinquish() {}
inline void tmem_dealloc(uint32_t, uint32_t) {}
inline void fence_before_sync() {}
inline void fence_after_sync() {}
inline void fence_async_smem() {}
inline const unsigned char *desc_elem(uint64_t desc, int r, int k) {
  const uint32_t start = (uint32_t)(desc & 0x3fffu) << 4;
  const uint32_t lbo = (uint32_t)((desc >> 16) & 0x3fffu) << 4, sbo = (uint32_t)((desc >> 32) & 0x3fffu) << 4;
  if (((desc >> 46) & 3u) != 1u || (desc >> 61) != 0u)
    emu::report_and_abort("matrix descriptor: not version 1 without swizzle");
  return emu::t_smem + start + (r >> 3) * sbo + (k >> 3) * lbo + (r & 7) * 16 + (k & 7) * 2;
}
inline void mma_host(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t accumulate) {
  const int n_dim = (int)((idesc >> 17) & 0x3fu) << 3, m_dim = (int)((idesc >> 24) & 0x1fu) << 4;
  if (((idesc >> 4) & 3u) != 1u || ((idesc >> 7) & 7u) != 1u || ((idesc >> 10) & 7u) != 1u || m_dim != 128)
    emu::report_and_abort("instruction descriptor: not bf16 x bf16 -> fp32 with M = 128");
  const int col0 = (int)(tmem_d & 0xffffu);
  if ((tmem_d >> 16) != 0u || col0 + n_dim > 512) emu::report_and_abort("MMA accumulator outside TMEM");
  for (int m = 0; m < m_dim; ++m)
    for (int n = 0; n < n_dim; ++n) {
      float acc = accumulate ? emu::t_tmem[m * 512 + col0 + n] : 0.f;
      for (int k = 0; k < 16; ++k) {
        const float x = bf16_lo(*reinterpret_cast<const uint16_t *>(desc_elem(adesc, m, k)));
        const float y = bf16_lo(*reinterpret_cast<const uint16_t *>(desc_elem(bdesc, n, k)));
        acc = std::fma(x, y, acc);
      }
      emu::t_tmem[m * 512 + col0 + n] = acc;
    }
}
inline void tmem_wait_ld() {}
}  // namespace umma
}  // namespace recsa
