"""The boundary from plain C: include/moe_b200.h compiles as C99 with
-Wall -Werror, and a C program linked against libmoe_b200.so gets the ABI
version, the launch count and the host-side argument checks (no GPU call)."""
import ctypes
import os
import subprocess
import textwrap

import pytest

import mixture_experts_layer_44_b200 as M

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = textwrap.dedent(r"""
    #include <stdio.h>
    #include <string.h>
    #include "moe_b200.h"

    int main(void) {
      int fails = 0;
      if (moe_abi_version() != 5) { puts("version"); ++fails; }
      if (moe_launch_count() != 0ull) { puts("launch count"); ++fails; }
      /* null x: rejected on the host before anything is enqueued */
      float logits[4];
      int r = moe_route(NULL, NULL, NULL, 4, 64, 8, 2, 1, MOE_BF16, logits, NULL, NULL, NULL,
                        NULL);
      if (r != MOE_ERR_INVALID_ARG || strstr(moe_last_error(), "moe_route") == NULL) {
        puts("route check"); ++fails;
      }
      /* nothing to do: OK without touching the GPU */
      int dummy[4];
      r = moe_experts((void*)dummy, dummy, NULL, (void*)dummy, (void*)dummy, 0, 256, 128, 4,
                      MOE_BF16, MOE_F16, (void*)dummy, (void*)dummy, NULL, 0, NULL, NULL);
      if (r != MOE_OK) { puts("experts N=0"); ++fails; }
      if (moe_dispatch_workspace_bytes(16384, 8, 128) < (size_t)64 * 128 * 4) {
        puts("dispatch ws"); ++fails;
      }
      /* the layer handle's descriptor, checked on the host */
      moe_layer_desc d;
      memset(&d, 0, sizeof d);
      d.T = 64; d.H = 256; d.E = 8; d.k = 2; d.I = 128; d.dtype = MOE_BF16; d.renormalize = 1;
      d.W_gate = dummy; d.w13 = dummy; d.w2 = dummy;
      size_t need = moe_layer_workspace_bytes(&d);
      if (need < (size_t)4 * 64 * 256 * 2) { puts("layer ws"); ++fails; }
      d.I = 100;
      if (moe_layer_workspace_bytes(&d) != 0) { puts("layer desc check"); ++fails; }
      moe_layer* L = NULL;
      if (moe_layer_create(&d, NULL, need, NULL, &L) != MOE_ERR_INVALID_ARG || L != NULL) {
        puts("layer create check"); ++fails;
      }
      /* the page's length-mismatch rule, on the host */
      r = moe_ep_partition((const int32_t*)dummy, 3, (const float*)dummy, 4, 2, 2, 0, 256,
                           dummy, dummy, (float*)dummy, dummy, dummy, (float*)dummy, dummy,
                           NULL, 0, NULL);
      if (r != MOE_ERR_INVALID_ARG || strcmp(moe_last_error(), "gate_indices length mismatch")) {
        puts("ep length"); ++fails;
      }
      r = moe_ep_partition((const int32_t*)dummy, 4, (const float*)dummy, 3, 2, 2, 0, 256,
                           dummy, dummy, (float*)dummy, dummy, dummy, (float*)dummy, dummy,
                           NULL, 0, NULL);
      if (r != MOE_ERR_INVALID_ARG || strcmp(moe_last_error(), "gate_weights length mismatch")) {
        puts("ep weights length"); ++fails;
      }
      printf("%s\n", fails ? "FAIL" : "OK");
      return fails;
    }
""")


def test_header_is_c99_and_the_library_links_from_c(tmp_path):
    if not os.path.exists(M.lib_path()):
        from mixture_experts_layer_44_b200 import build
        build.build()
    src = tmp_path / "abi_check.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "abi_check"
    lib_dir = os.path.dirname(M.lib_path())
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
           str(src), "-o", str(exe), "-L", lib_dir, "-lmoe_b200", f"-Wl,-rpath,{lib_dir}"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0 and "cannot find -lmoe_b200" in r.stderr:
        pytest.skip("libmoe_b200.so not linkable here")
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and r.stdout.strip().endswith("OK"), r.stdout + r.stderr


def test_layer_descriptor_layout_matches_the_binding(tmp_path):
    # the ctypes mirror of moe_layer_desc must have the C struct's size and offsets
    fields = [f for f, _ in M.MoELayerDesc._fields_]
    body = "\n".join(f'  printf("{f} %zu\\n", offsetof(moe_layer_desc, {f}));' for f in fields)
    src = tmp_path / "desc_layout.c"
    src.write_text(textwrap.dedent("""\
        #include <stddef.h>
        #include <stdio.h>
        #include "moe_b200.h"
        int main(void) {
          printf("sizeof %zu\\n", sizeof(moe_layer_desc));
        """) + body + "\n  return 0;\n}\n")
    exe = tmp_path / "desc_layout"
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                        str(src), "-o", str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    out = dict(l.split() for l in subprocess.run([str(exe)], capture_output=True, text=True,
                                                 timeout=60).stdout.splitlines())
    assert int(out["sizeof"]) == ctypes.sizeof(M.MoELayerDesc)
    for f in fields:
        assert int(out[f]) == getattr(M.MoELayerDesc, f).offset, f
