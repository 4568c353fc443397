"""Cut kernels out of the library's sources, unchanged apart from the shared-memory
declarations and inline PTX, for compiling on the host against emu_cuda.h: the lean attend
kernel (and the helpers it uses) and the append kernel.  Test infrastructure."""

from __future__ import annotations

import re


def extract_lean(src_path: str, out_path: str) -> None:
    lines = open(src_path).read().split("\n")

    def idx(pat: str) -> int:
        for i, line in enumerate(lines):
            if pat in line:
                return i
        raise ValueError(f"marker not found in the attend source: {pat}")

    head = lines[: idx("// ------------------------------------------------------------------ warp-level selection")]
    ws0 = idx("__device__ __forceinline__ bool workspace_ok")
    ws1 = idx("// ================================================================== CTA / cluster kernel")
    align = idx("__host__ __device__ inline int align128")
    lean0 = idx("// ================================================================== lean cluster kernel")
    lean1 = idx("// ================================================================== warp-per-tile kernel")
    text = "\n".join(head + lines[ws0:ws1] + [lines[align]] + lines[lean0:lean1] +
                     ["}  // namespace", "}  // namespace recsa"])
    for old, new in (("#include <cooperative_groups.h>", ""), ("#include <cuda_runtime.h>", ""),
                     ('#include "recsa_device.cuh"', '#include "emu_device.h"'),
                     ("namespace cg = cooperative_groups;", ""),
                     ("extern __shared__ __align__(128) unsigned char smem[];", "unsigned char *smem = emu::t_smem;")):
        if old not in text:
            raise ValueError(f"expected text not found in the attend source: {old}")
        text = text.replace(old, new)
    text = re.sub(r"__device__ __forceinline__ uint2 ld_nc_u2\(const void \*p\) \{.*?\n\}",
                  "inline uint2 ld_nc_u2(const void *p) { return *reinterpret_cast<const uint2 *>(p); }", text,
                  flags=re.S)
    text = re.sub(r"__device__ __forceinline__ float4 ld_nc_f4\(const void \*p\) \{.*?\n\}",
                  "inline float4 ld_nc_f4(const void *p) { return *reinterpret_cast<const float4 *>(p); }", text,
                  flags=re.S)
    open(out_path, "w").write(text)


def extract_umma(src_path: str, out_path: str) -> None:
    """recsa_umma.cuh with its inline-PTX helpers (TMEM, MMA, commit, fences, TMEM loads)
    replaced by host versions from emu_umma_ops.h; the operand layout, the descriptors, the
    split into bf16 parts and the order of the products stay the library's own."""
    text = open(src_path).read()
    text = text.replace('#include "recsa_device.cuh"', '#include "emu_device.h"\n#include "emu_umma_ops.h"')
    for fn in ("void tmem_alloc", "void tmem_relinquish", "void tmem_dealloc", "void fence_before_sync",
               "void fence_after_sync", "void fence_async_smem", "void tmem_wait_ld"):
        pat = r"__device__ __forceinline__ " + re.escape(fn) + r"\(.*?(\n\}|\); \}|::: \"memory\"\); \})"
        text, k = re.subn(pat, "", text, count=1, flags=re.S)
        if k != 1:
            raise ValueError(f"helper not found in the tcgen05 header: {fn}")
    text, k = re.subn(r"__device__ __forceinline__ void mma\(uint32_t tmem_d, .*?\n\}",
                      "inline void mma(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,\n"
                      "                uint32_t accumulate) {\n"
                      "  mma_host(tmem_d, adesc, bdesc, idesc, accumulate);\n}", text, count=1, flags=re.S)
    if k != 1:
        raise ValueError("mma not found in the tcgen05 header")
    text, k = re.subn(r"__device__ __forceinline__ void commit\(uint64_t \*bar\) \{.*?\n\}",
                      "inline void commit(uint64_t *bar) { mbar_arrive(bar); }", text, count=1, flags=re.S)
    if k != 1:
        raise ValueError("commit not found in the tcgen05 header")
    text, k = re.subn(r"__device__ __forceinline__ void tmem_ld32\(uint32_t taddr, uint32_t \(&v\)\[32\]\) \{.*?\n\}",
                      "inline void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {\n"
                      "  const int lane = (int)(taddr >> 16) + (emu::t_tid & 31), col = (int)(taddr & 0xffffu);\n"
                      "  for (int i = 0; i < 32; ++i) std::memcpy(&v[i], &emu::t_tmem[lane * 512 + col + i], 4);\n}",
                      text, count=1, flags=re.S)
    if k != 1:
        raise ValueError("tmem_ld32 not found in the tcgen05 header")
    open(out_path, "w").write(text)


def extract_extend(src_path: str, out_path: str) -> None:
    """The build source up to the end of the append kernel (one CTA per (sequence, head)),
    with recsa_umma.cuh taken from the extracted copy next to `out_path`."""
    import os

    text = open(src_path).read()
    end = text.index("// k_new / v_new [B][C][Hkv][128] -> token caches")
    text = text[:end] + "}  // namespace\n}  // namespace recsa\n"
    extract_umma(os.path.join(os.path.dirname(src_path), "recsa_umma.cuh"),
                 os.path.join(os.path.dirname(out_path), "umma_extracted.h"))
    for old, new in (("#include <cuda_runtime.h>", ""), ('#include "recsa_device.cuh"', '#include "emu_device.h"'),
                     ('#include "recsa_umma.cuh"', '#include "umma_extracted.h"'),
                     ('asm volatile("prefetch.global.L2 [%0];" ::"l"(p));', "(void)p;"),
                     ('asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");',
                      "(void)p;\n  (void)bytes;")):
        if old not in text:
            raise ValueError(f"expected text not found in the build source: {old}")
        text = text.replace(old, new)
    decl = "extern __shared__ __align__(128) unsigned char smem_u8[];"
    if text.count(decl) < 1:
        raise ValueError("shared-memory declaration not found in the build source")
    text = text.replace(decl, "unsigned char *smem_u8 = emu::t_smem;")
    open(out_path, "w").write(text)
