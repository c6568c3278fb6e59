"""Host-side checks of the C-ABI library (no GPU): it loads, exports every symbol the header
declares, its structs match the ctypes mirror byte for byte, and invalid arguments are rejected
with the documented status before anything is launched."""
import ctypes
import os
import re
import subprocess


import oracle as O
import block_scaled_bit_rht16_b200 as fq
from block_scaled_bit_rht16_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fp4q.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(fp4q_[a-z0-9_]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    lib = _lib.load()
    names = _declared()
    assert names == sorted(_lib.EXPORTS)
    for n in names:
        assert hasattr(lib, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", _lib.LIB_PATH], capture_output=True, text=True).stdout
    for n in names:
        assert re.search(r"\bT %s$" % n, out, flags=re.M), n


def test_struct_layout_matches_header(tmp_path):
    prog = tmp_path / "layout.c"
    prog.write_text('''#include <stdio.h>
#include <stddef.h>
#include "fp4q.h"
int main(void) {
  printf("%zu %zu %zu %zu %zu\\n", sizeof(fp4q_config), offsetof(fp4q_config, sr_seed),
         offsetof(fp4q_config, outputs), sizeof(fp4q_stats_t), offsetof(fp4q_stats_t, status));
  return 0;
}''')
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(prog), "-o", str(exe)], check=True)
    got = [int(v) for v in subprocess.run([str(exe)], capture_output=True, text=True).stdout.split()]
    want = [ctypes.sizeof(_lib.fp4q_config), _lib.fp4q_config.sr_seed.offset,
            _lib.fp4q_config.outputs.offset, ctypes.sizeof(_lib.fp4q_stats_t),
            _lib.fp4q_stats_t.status.offset]
    assert got == want


def test_status_strings():
    lib = _lib.load()
    for s in range(8):
        assert lib.fp4q_status_string(s)
    assert lib.fp4q_status_string(0) == b"ok"
    assert lib.fp4q_status_string(99) == b"unknown status"


def test_sign_mask_from_seed_matches_oracle():
    for seed in (0, 1, 0x5EED0001, 0x5EED0005, 2**63 + 17):
        assert fq.sign_mask_from_seed(seed) == O.sign_mask_from_seed(seed)


def test_workspace_sizes():
    assert fq.workspace_size(fq.Config(), 128, 256) == 0
    base = fq.workspace_size(fq.Config(scale=fq.FP4Q_SCALE_E4M3_1x16_TENSOR, grid=fq.FP4Q_GRID_E2M1), 128, 256)
    assert base == 256
    st = fq.workspace_size(fq.Config(stats=True), 128, 256)
    assert st > 256 and st % 8 == 0
    assert fq.workspace_size(fq.Config(grid=fq.FP4Q_GRID_E2M1, scale=fq.FP4Q_SCALE_UE8M0_1x32), 1, 32) == 0


FAKE = 1 << 20   # a 256-byte-aligned non-null address; never dereferenced: validation fails first


def _q(cfg=None, x=FAKE, rows=4, cols=32, ld=32, codes=FAKE, scales=FAKE, ts=None, given=0,
       deq=None, ws=None, ws_bytes=0):
    lib = _lib.load()
    c = (cfg or fq.Config()).c()
    return lib.fp4q_rht_quantize(ctypes.byref(c), x, rows, cols, ld, codes, scales, ts, given, deq,
                                 ws, ws_bytes, None)


def test_rejects_bad_arguments_before_launch():
    assert _q(x=None) == _lib.FP4Q_ERR_INVALID_ARG
    assert _q(codes=None) == _lib.FP4Q_ERR_INVALID_ARG
    assert _q(cols=24, ld=24) == _lib.FP4Q_ERR_SHAPE
    assert _q(rows=-1) == _lib.FP4Q_ERR_SHAPE
    assert _q(ld=16) == _lib.FP4Q_ERR_SHAPE
    assert _q(ld=36) == _lib.FP4Q_ERR_ALIGN
    assert _q(x=FAKE + 8) == _lib.FP4Q_ERR_ALIGN
    assert _q(codes=FAKE + 4) == _lib.FP4Q_ERR_ALIGN
    assert _q(fq.Config(dequant=True)) == _lib.FP4Q_ERR_INVALID_ARG          # dequant requested, NULL
    assert _q(fq.Config(stats=True)) == _lib.FP4Q_ERR_WORKSPACE              # stats need a workspace
    assert _q(fq.Config(stats=True), ws=FAKE, ws_bytes=100) == _lib.FP4Q_ERR_WORKSPACE
    assert _q(fq.Config(stats=True), ws=FAKE + 64, ws_bytes=1 << 20) == _lib.FP4Q_ERR_ALIGN
    e4 = fq.Config(grid=fq.FP4Q_GRID_E2M1, scale=fq.FP4Q_SCALE_E4M3_1x16_TENSOR)
    assert _q(e4) == _lib.FP4Q_ERR_INVALID_ARG                               # tensor scale missing
    assert _q(e4, ts=FAKE) == _lib.FP4Q_ERR_WORKSPACE                        # amax pass needs one
    assert _q(fq.Config(grid=7)) == _lib.FP4Q_ERR_INVALID_ARG
    assert _q(fq.Config(scale=9)) == _lib.FP4Q_ERR_INVALID_ARG
    assert _q(fq.Config(round=2)) == _lib.FP4Q_ERR_INVALID_ARG
    assert _q(fq.Config(rht=2)) == _lib.FP4Q_ERR_INVALID_ARG
    assert _q(fq.Config(sign_mask=1 << 16)) == _lib.FP4Q_ERR_INVALID_ARG
    assert _q(fq.Config(grid=fq.FP4Q_GRID_IF4)) == _lib.FP4Q_ERR_UNSUPPORTED  # IF4 needs E4M3
    assert _q(fq.Config(grid=fq.FP4Q_GRID_E1M2, scale=fq.FP4Q_SCALE_UE8M0_1x32)) == _lib.FP4Q_ERR_UNSUPPORTED
    mx = fq.Config(grid=fq.FP4Q_GRID_E2M1, scale=fq.FP4Q_SCALE_UE8M0_1x32)
    assert _q(mx, cols=48, ld=48) == _lib.FP4Q_ERR_SHAPE
    assert _q(mx, codes=FAKE + 8) == _lib.FP4Q_ERR_ALIGN
    for bad in (1, 5, 6, 7):   # e2m1_max takes 0, 4, 3, 2
        c = fq.Config(grid=fq.FP4Q_GRID_E2M1).c()
        c.e2m1_max = bad
        assert _lib.load().fp4q_rht_quantize(ctypes.byref(c), FAKE, 4, 32, 32, FAKE, FAKE, None, 0,
                                             None, None, 0, None) == _lib.FP4Q_ERR_INVALID_ARG
    # block-scaled MMA scale layout: E4M3 / UE8M0 scales only, 128-row and 4-column tiles
    nvm = fq.Config(grid=fq.FP4Q_GRID_E2M1, scale=fq.FP4Q_SCALE_E4M3_1x16_TENSOR, mma_scales=True)
    assert _q(fq.Config(mma_scales=True)) == _lib.FP4Q_ERR_UNSUPPORTED          # FP32 scales
    assert _q(fq.Config(grid=fq.FP4Q_GRID_IF4, scale=fq.FP4Q_SCALE_E4M3_1x16_TENSOR,
                        mma_scales=True), ts=FAKE) == _lib.FP4Q_ERR_UNSUPPORTED
    assert _q(nvm, rows=4, cols=64, ld=64, ts=FAKE) == _lib.FP4Q_ERR_SHAPE        # rows % 128
    assert _q(nvm, rows=128, cols=32, ld=32, ts=FAKE) == _lib.FP4Q_ERR_SHAPE      # 2 scale columns
    # range restriction is for E2M1 with the FP32 1x16 scale only
    assert _q(fq.Config(grid=fq.FP4Q_GRID_E1M2, e2m1_max=4)) == _lib.FP4Q_ERR_UNSUPPORTED
    assert _q(fq.Config(grid=fq.FP4Q_GRID_E2M1, scale=fq.FP4Q_SCALE_E4M3_1x16_TENSOR,
                        e2m1_max=3)) == _lib.FP4Q_ERR_UNSUPPORTED
    assert _q(fq.Config(grid=fq.FP4Q_GRID_E2M1, scale=fq.FP4Q_SCALE_UE8M0_1x32,
                        e2m1_max=2)) == _lib.FP4Q_ERR_UNSUPPORTED
    assert _lib.load().fp4q_rht_quantize(None, FAKE, 4, 32, 32, FAKE, FAKE, None, 0, None, None, 0,
                                         None) == _lib.FP4Q_ERR_INVALID_ARG


def test_dual_dequant_rht_stats_validation():
    lib = _lib.load()
    r, c = fq.Config(round=fq.FP4Q_ROUND_SR).c(), fq.Config(round=fq.FP4Q_ROUND_SR, sr_stream=1).c()
    dual = lambda rc=r, cc=c, M=32, N=32, ld=32, dy=FAKE, cr=FAKE: lib.fp4q_quantize_dual(
        ctypes.byref(rc), ctypes.byref(cc), dy, M, N, ld, cr, FAKE, FAKE, FAKE, None, 0, None)
    assert dual(M=24) == _lib.FP4Q_ERR_SHAPE
    assert dual(N=40, ld=40) == _lib.FP4Q_ERR_SHAPE
    assert dual(M=2 ** 31) == _lib.FP4Q_ERR_SHAPE
    assert dual(N=2 ** 31, ld=2 ** 31) == _lib.FP4Q_ERR_SHAPE
    assert dual(M=2 ** 24, N=2 ** 24, ld=2 ** 24) == _lib.FP4Q_ERR_SHAPE   # 2^35 tiles: one CTA each
    assert dual(dy=None) == _lib.FP4Q_ERR_INVALID_ARG
    assert dual(cr=FAKE + 4) == _lib.FP4Q_ERR_ALIGN
    e2 = fq.Config(grid=fq.FP4Q_GRID_E2M1).c()
    assert dual(cc=e2) == _lib.FP4Q_ERR_UNSUPPORTED
    nv = fq.Config(scale=fq.FP4Q_SCALE_E4M3_1x16_TENSOR).c()
    assert dual(rc=nv) == _lib.FP4Q_ERR_UNSUPPORTED
    assert dual(rc=fq.Config(dequant=True).c()) == _lib.FP4Q_ERR_UNSUPPORTED
    r4 = fq.Config(grid=fq.FP4Q_GRID_E2M1, round=fq.FP4Q_ROUND_SR, e2m1_max=4).c()
    c4 = fq.Config(grid=fq.FP4Q_GRID_E2M1, round=fq.FP4Q_ROUND_SR, sr_stream=1, e2m1_max=4).c()
    assert dual(rc=r4, cc=c4) == _lib.FP4Q_ERR_UNSUPPORTED
    d = fq.Config().c()
    assert lib.fp4q_dequantize(ctypes.byref(d), None, FAKE, None, 4, 32, 0, FAKE, None) == _lib.FP4Q_ERR_INVALID_ARG
    assert lib.fp4q_dequantize(ctypes.byref(d), FAKE, FAKE, None, 4, 24, 0, FAKE, None) == _lib.FP4Q_ERR_SHAPE
    assert lib.fp4q_dequantize(ctypes.byref(d), FAKE, FAKE, None, 4, 32, 2, FAKE, None) == _lib.FP4Q_ERR_INVALID_ARG
    assert lib.fp4q_dequantize(ctypes.byref(nv), FAKE, FAKE, None, 4, 32, 0, FAKE, None) == _lib.FP4Q_ERR_INVALID_ARG
    assert lib.fp4q_rht16(FAKE, 4, 24, 24, 0, FAKE, 0, None) == _lib.FP4Q_ERR_SHAPE
    assert lib.fp4q_rht16(FAKE, 4, 32, 32, 1 << 17, FAKE, 0, None) == _lib.FP4Q_ERR_INVALID_ARG
    assert lib.fp4q_rht16(FAKE + 2, 4, 32, 32, 0, FAKE, 0, None) == _lib.FP4Q_ERR_ALIGN
    st = _lib.fp4q_stats_t()
    assert lib.fp4q_stats(None, 0, ctypes.byref(st), None) == _lib.FP4Q_ERR_INVALID_ARG
    assert lib.fp4q_stats(FAKE, 256, ctypes.byref(st), None) == _lib.FP4Q_ERR_WORKSPACE


def test_recipe_presets():
    # UFP4 recipe table: rotation on every path, SR on dY only; E2M1 baseline: rotation on bwd_dw
    for path in ("fwd_y", "bwd_dx", "bwd_dw"):
        u = fq.recipe("ufp4", path, "x", sign_mask=0x1234)
        assert u.grid == fq.FP4Q_GRID_E1M2 and u.rht == 1 and u.round == fq.FP4Q_ROUND_RTNE
        e = fq.recipe("e2m1", path, "x", sign_mask=0x1234)
        assert e.grid == fq.FP4Q_GRID_E2M1 and e.rht == (1 if path == "bwd_dw" else 0)
    dy = fq.recipe("ufp4", "bwd_dw", "dy", sr_seed=5)
    assert dy.round == fq.FP4Q_ROUND_SR and dy.sr_stream == 1
    assert fq.recipe("ufp4", "bwd_dx", "dy").sr_stream == 0


def test_grouped_validation():
    lib = _lib.load()
    nv = fq.Config(grid=fq.FP4Q_GRID_E2M1, scale=fq.FP4Q_SCALE_E4M3_1x16_TENSOR).c()
    assert lib.fp4q_grouped_workspace_size(ctypes.byref(nv), 64) == 256
    assert lib.fp4q_grouped_workspace_size(ctypes.byref(nv), 65) == 512
    assert lib.fp4q_grouped_workspace_size(ctypes.byref(nv), 0) == 0
    assert lib.fp4q_grouped_workspace_size(ctypes.byref(fq.Config().c()), 64) == 0   # FP32 scales

    def g(cfg=nv, offs=FAKE, n=4, ts=FAKE, given=0, ws=FAKE, wsb=256, rows=4, cols=32):
        return lib.fp4q_rht_quantize_grouped(ctypes.byref(cfg), FAKE, rows, cols, cols, offs, n, FAKE,
                                             FAKE, ts, given, ws, wsb, None)
    assert g(n=0) == _lib.FP4Q_ERR_INVALID_ARG
    assert g(n=(1 << 24) + 1) == _lib.FP4Q_ERR_INVALID_ARG
    assert g(offs=None) == _lib.FP4Q_ERR_INVALID_ARG
    assert g(ts=None) == _lib.FP4Q_ERR_INVALID_ARG
    assert g(given=2) == _lib.FP4Q_ERR_INVALID_ARG
    assert g(offs=FAKE + 4) == _lib.FP4Q_ERR_ALIGN
    assert g(ws=None) == _lib.FP4Q_ERR_WORKSPACE
    assert g(wsb=128) == _lib.FP4Q_ERR_WORKSPACE
    assert g(cols=24) == _lib.FP4Q_ERR_SHAPE
    deq = fq.Config(grid=fq.FP4Q_GRID_E2M1, scale=fq.FP4Q_SCALE_E4M3_1x16_TENSOR, dequant=True).c()
    assert g(cfg=deq) == _lib.FP4Q_ERR_UNSUPPORTED
    sr = fq.Config(grid=fq.FP4Q_GRID_E2M1, scale=fq.FP4Q_SCALE_E4M3_1x16_TENSOR,
                   round=fq.FP4Q_ROUND_SR).c()
    assert g(cfg=sr) == _lib.FP4Q_ERR_UNSUPPORTED


def test_plain_c_program_uses_the_library(tmp_path):
    # the ABI is usable from C alone: a program built against include/fp4q.h and linked with
    # libfp4q.so calls the host-side entry points and gets the documented statuses (no GPU work:
    # every quantize call here is rejected by validation)
    prog = tmp_path / "consumer.c"
    prog.write_text(r'''#include <stdio.h>
#include <string.h>
#include "fp4q.h"
int main(void) {
  fp4q_config c;
  memset(&c, 0, sizeof c);
  c.grid = FP4Q_GRID_E1M2; c.scale = FP4Q_SCALE_FP32_1x16; c.round = FP4Q_ROUND_RTNE; c.rht = 1;
  c.sign_mask = fp4q_sign_mask_from_seed(7); c.outputs = FP4Q_OUT_CODES;
  void* fake = (void*)(uintptr_t)(1u << 20);
  printf("%u\n", c.sign_mask);
  printf("%zu\n", fp4q_workspace_size(&c, 128, 256));
  c.outputs |= FP4Q_OUT_STATS;
  printf("%zu\n", fp4q_workspace_size(&c, 128, 256));
  c.outputs = FP4Q_OUT_CODES;
  printf("%d\n", (int)fp4q_rht_quantize(&c, fake, 4, 24, 24, fake, fake, NULL, 0, NULL, NULL, 0, NULL));
  printf("%d\n", (int)fp4q_rht_quantize(&c, NULL, 4, 32, 32, fake, fake, NULL, 0, NULL, NULL, 0, NULL));
  printf("%d\n", (int)fp4q_quantize_dual(&c, &c, fake, 24, 32, 32, fake, fake, fake, fake, NULL, 0, NULL));
  printf("%d\n", (int)fp4q_rht_quantize_noalloc(&c, (char*)fake + 8, 4, 32, 32, fake, fake, NULL, 0, NULL, NULL));
  printf("%s\n", fp4q_status_string(FP4Q_ERR_ALIGN));
  return 0;
}
''')
    exe = tmp_path / "consumer"
    libdir = os.path.dirname(_lib.LIB_PATH)
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(prog),
                    "-L", libdir, "-lfp4q", "-Wl,-rpath," + libdir, "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split("\n")
    assert int(out[0]) == O.sign_mask_from_seed(7)
    assert int(out[1]) == 0 and int(out[2]) == fq.workspace_size(fq.Config(stats=True), 128, 256)
    assert [int(v) for v in out[3:7]] == [_lib.FP4Q_ERR_SHAPE, _lib.FP4Q_ERR_INVALID_ARG,
                                          _lib.FP4Q_ERR_SHAPE, _lib.FP4Q_ERR_ALIGN]
    assert out[7] == "misaligned pointer or row pitch"


def test_binding_rejects_host_tensors_before_any_call():
    # every public function checks its tensors first: host memory never reaches the library
    import pytest
    import torch
    x = torch.zeros((4, 32), dtype=torch.bfloat16)
    cfg = fq.Config()
    with pytest.raises(TypeError):
        fq.rht_quantize(cfg, x)
    with pytest.raises(TypeError):
        fq.rht_quantize_grouped(cfg, x, torch.tensor([0, 4]))
    with pytest.raises(TypeError):
        fq.quantize_dual(cfg, cfg, torch.zeros((16, 32), dtype=torch.bfloat16))
    with pytest.raises(TypeError):
        fq.dequantize(cfg, torch.zeros((4, 16), dtype=torch.uint8), torch.zeros((4, 2)))
    with pytest.raises(TypeError):
        fq.rht16(x, 0)
    with pytest.raises(TypeError):
        fq.tensor_scale(fq.Config(scale=fq.FP4Q_SCALE_E4M3_1x16_TENSOR), x)
    with pytest.raises(TypeError):
        fq.stats(torch.zeros(256, dtype=torch.uint8))
    with pytest.raises(TypeError):
        fq.rht_quantize(cfg, torch.zeros((4, 32), dtype=torch.float32))


def test_gemm_validation():
    lib = _lib.load()
    g = lambda M=128, N=128, K=256, ldo=128, a=FAKE, sa=FAKE, out=FAKE, ts=FAKE: lib.fp4q_gemm_nvfp4(
        a, sa, ts, FAKE, FAKE, FAKE, M, N, K, out, ldo, None)
    assert g(M=100) == _lib.FP4Q_ERR_SHAPE            # M not a multiple of 128
    assert g(N=64) == _lib.FP4Q_ERR_SHAPE
    assert g(K=128) == _lib.FP4Q_ERR_SHAPE            # K not a multiple of 256
    assert g(K=0) == _lib.FP4Q_ERR_SHAPE
    assert g(ldo=64) == _lib.FP4Q_ERR_SHAPE           # ldo < N
    assert g(M=65536 * 128) == _lib.FP4Q_ERR_SHAPE    # beyond the tile grid's y limit
    assert g(M=65535 * 128, N=(1 << 16) * 128, ldo=(1 << 16) * 128) == _lib.FP4Q_ERR_SHAPE   # over 2^30 tiles
    assert g(a=None) == _lib.FP4Q_ERR_INVALID_ARG
    assert g(ts=None) == _lib.FP4Q_ERR_INVALID_ARG
    assert g(a=FAKE + 8) == _lib.FP4Q_ERR_ALIGN       # codes 16-byte aligned
    assert g(sa=FAKE + 4) == _lib.FP4Q_ERR_ALIGN
    assert g(ldo=132) == _lib.FP4Q_ERR_ALIGN          # 16-byte output rows
    assert g(M=1 << 16, K=1 << 31) == _lib.FP4Q_ERR_SHAPE   # over 2^31 - 1 scale tiles
    assert g(M=0) == _lib.FP4Q_OK                     # empty: nothing to do
    mx = lambda M=128, N=128, K=256, ldo=128, a=FAKE, sa=FAKE, out=FAKE: lib.fp4q_gemm_mxfp4(
        a, sa, FAKE, FAKE, M, N, K, out, ldo, None)
    assert mx(M=100) == _lib.FP4Q_ERR_SHAPE
    assert mx(K=128) == _lib.FP4Q_ERR_SHAPE
    assert mx(ldo=64) == _lib.FP4Q_ERR_SHAPE
    assert mx(sa=None) == _lib.FP4Q_ERR_INVALID_ARG
    assert mx(sa=FAKE + 4) == _lib.FP4Q_ERR_ALIGN
    assert mx(M=0) == _lib.FP4Q_OK
