"""include/moe.h is a plain C header: a C99 translation unit and a C++17 one
that include it and call every entry point compile without warnings, and the
C object links against the built libmoe.so (nothing is run)."""
import os
import shutil
import subprocess

import pytest

from quantized_mixture_experts_sigmoid_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
OUT = os.path.join(ROOT, "quantized_mixture_experts_sigmoid_b200", "_build")

SRC = r"""
#include "moe.h"
#include <stddef.h>

int use_every_entry_point(void* p, moe_stream_t s) {
    moe_router_cfg cfg = {256, 8, 4, 8, 2.5f, 0.0f};
    moe_experts ex = {MOE_Q_INT4, 256, 6144, 2048, 0, 0, 0, 0, 0, 0, 0};
    int st = 0, n = 0;
    double ms = 0.0;
    size_t b = moe_route_workspace_bytes(1, &cfg) + moe_expert_ffn_workspace_bytes(&ex, 1, 8) +
               moe_layer_workspace_bytes(1, &cfg, &ex, NULL);
    int rc = moe_route((const uint16_t*)p, 1, 6144, (const float*)p, (const float*)p, &cfg, (int32_t*)p,
                       (float*)p, p, b, s);
    rc |= moe_route_noalloc((const uint16_t*)p, 1, 6144, (const float*)p, (const float*)p, &cfg, (int32_t*)p,
                            (float*)p, s);
    rc |= moe_union((const int32_t*)p, 1, 8, 256, (int32_t*)p, (int32_t*)p, (int32_t*)p, (int32_t*)p, (int32_t*)p,
                    NULL, NULL, s);
    rc |= moe_quantize_q8_0(p, MOE_OUT_BF16, 1, 6144, (int8_t*)p, (float*)p, s);
    rc |= moe_usage_accumulate((const int32_t*)p, 1, 8, 256, (uint32_t*)p, s);
    rc |= moe_usage_rank((const uint32_t*)p, 256, (int32_t*)p, s);
    rc |= moe_expert_ffn_q(&ex, (const uint16_t*)p, 1, 1, NULL, NULL, NULL, NULL, NULL, (float*)p, p, b, s);
    rc |= moe_combine((const float*)p, (const float*)p, NULL, 1, 8, 6144, p, MOE_OUT_F32, s);
    rc |= moe_layer_forward((const uint16_t*)p, 1, (const float*)p, (const float*)p, &cfg, &ex, NULL, p,
                            MOE_OUT_BF16, NULL, NULL, p, b, s);
    rc |= moe_layer_path(1, &cfg, &ex, NULL);
    rc |= moe_workspace_status(p, 1, &st, s);
    rc |= moe_workspace_set_wait_limit(p, 0, s);
    rc |= moe_profile_enable(0) | moe_profile_read(&ms, &n);
    return rc + (int)moe_launch_count() + (moe_strerror(rc)[0] != 0) + (moe_cuda_error_string()[0] != 0);
}
"""


@pytest.mark.parametrize("lang", ["c", "c++"])
def test_header_compiles_and_links(lang):
    compiler = "gcc" if lang == "c" else "g++"
    if shutil.which(compiler) is None:
        pytest.skip(f"no {compiler}")
    os.makedirs(OUT, exist_ok=True)
    tag = f"{os.getpid()}_{lang.replace('+', 'x')}"
    src = os.path.join(OUT, f"header_check_{tag}.{'c' if lang == 'c' else 'cpp'}")
    obj = os.path.join(OUT, f"header_check_{tag}.o")
    exe = os.path.join(OUT, f"header_check_{tag}")
    std = "-std=c99" if lang == "c" else "-std=c++17"
    try:
        with open(src, "w") as f:
            f.write(SRC + ("\nint main(void) { return use_every_entry_point(0, 0) == 12345; }\n"))
        r = subprocess.run([compiler, std, "-Wall", "-Wextra", "-Werror", "-c", "-I", os.path.join(ROOT, "include"),
                            src, "-o", obj], capture_output=True, text=True)
        assert r.returncode == 0, r.stderr
        if lang == "c":
            lib = B.build()
            r = subprocess.run([compiler, obj, "-o", exe, lib, "-Wl,--unresolved-symbols=ignore-in-shared-libs"],
                               capture_output=True, text=True)
            assert r.returncode == 0, r.stderr
    finally:
        for path in (src, obj, exe):
            if os.path.exists(path):
                os.remove(path)
