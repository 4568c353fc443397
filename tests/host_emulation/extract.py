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


def extract_extend(src_path: str, out_path: str) -> None:
    """The build source up to the end of the append kernel (one CTA per (sequence, head))."""
    text = open(src_path).read()
    end = text.index("// k_new / v_new [B][C][Hkv][128] -> token caches")
    text = text[:end] + "}  // namespace\n}  // namespace recsa\n"
    for old, new in (("#include <cuda_runtime.h>", ""), ('#include "recsa_device.cuh"', '#include "emu_device.h"'),
                     ('asm volatile("prefetch.global.L2 [%0];" ::"l"(p));', "(void)p;")):
        if old not in text:
            raise ValueError(f"expected text not found in the build source: {old}")
        text = text.replace(old, new)
    decl = "extern __shared__ __align__(16) float smem_f[];"
    if text.count(decl) < 1:
        raise ValueError("shared-memory declaration not found in the build source")
    text = text.replace(decl, "float *smem_f = reinterpret_cast<float *>(emu::t_smem);")
    open(out_path, "w").write(text)
