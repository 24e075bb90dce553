"""The bounds-checked build (libvmla_checked.so, VMLA_CHECKED=1), run in a child process: every
computed global store of the tensor-core kernels is tested against its buffer's extent.  Every call of
the path, the dense layer, the rewrite, the row-range (sharded) calls, the executor, the key-split
kernels (d_c 64 / 128) and the paired-CTA compress (Wan shapes, B = 4) must run with no store outside
its buffer; with the recorded extents shortened by one 32-column chunk
(vmla_debug_shrink_extents) the stores at the buffers' ends must be reported instead (and skipped)."""
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIB = os.path.join(ROOT, "rank_latent_kv_vmla_b200", "libvmla_checked.so")

SCRIPT = r"""
import sys, torch
sys.path.insert(0, ROOT); sys.path.insert(0, ROOT + "/tests")
from rank_latent_kv_vmla_b200 import vmla as V
from rank_latent_kv_vmla_b200.sharding import token_shards
import synthetic
from parity import MID
assert V.LIB.vmla_debug_shrink_extents(0) == 1, "not a checked build"
dev = "cuda"
cfg, B = MID, 2
w, wuk, wuv = (t.to(dev) for t in synthetic.draw_weights(cfg, 3))
w_kv = synthetic.draw_dense_weights(cfg, 4).to(dev)
lc = V.LatentCache(cfg, B, device=dev)
dc = V.DenseCache(cfg, B, device=dev)
reps = [V.LatentCache(cfg, B, device=dev) for _ in range(3)]
shards = token_shards(cfg.chunk_tokens, 3, align=8)        # 120 tokens: 40 + 40 + 40
def status(what):
    code = V.device_status()
    print(what, code)
    return code
for k in range(4):                       # the ring wraps: every slot, the last rows included, written
    x, qn, qr = (t.to(dev) for t in synthetic.draw_chunk(cfg, B, 10 + k))
    f0 = lc.frames_written
    V.compress_append(cfg, x, w, lc)
    V.compress_rewrite(cfg, x, w, lc)
    q_abs = V.absorb_q(cfg, qn, qr, wuk, f0)
    o_lat, lse = V.latent_attention(cfg, q_abs, lc, f0, want_lse=True)
    V.value_up(cfg, o_lat, wuv)
    V.latent_attention_fused(cfg, qn, qr, wuk, wuv, lc, f0, want_lse=True)
    V.dense_append(cfg, x, w_kv, dc)
    V.dense_mha(cfg, V.rope_q(cfg, qn, qr, f0), dc, f0, want_lse=True)
    for b0, n in shards:
        V.compress_append_rows(cfg, x[:, b0:b0 + n].contiguous(), w, f0, b0, [r.struct for r in reps], B)
    for r in reps:
        r.struct.frames_written = f0 + cfg.chunk_frames
    for g, (b0, n) in enumerate(shards):
        V.latent_attention_fused_rows(cfg, qn[:, b0:b0 + n].contiguous(), qr[:, b0:b0 + n].contiguous(), wuk, wuv,
                                      reps[g], f0, b0, want_lse=True)
    assert status(f"chunk {k}") == 0
with V.Executor(cfg, B) as ex:
    hosts = [t.pin_memory() for t in synthetic.draw_chunk(cfg, B, 20)]
    ho = torch.empty((B, cfg.chunk_tokens, cfg.n_heads, cfg.d_v), dtype=torch.bfloat16).pin_memory()
    for _ in range(3):
        ex.submit(lc, w, wuk, wuv, *hosts, ho)
    ex.wait()
assert status("executor") == 0
# the key-split attention kernels (d_c 64 / 128) and the paired-CTA compress (Wan shapes at B = 4)
from rank_latent_kv_vmla_b200.config import WAN
for d_c in (64, 128):
    c2 = MID.replace(d_c=d_c)
    w2, wuk2, wuv2 = (t.to(dev) for t in synthetic.draw_weights(c2, 5))
    l2 = V.LatentCache(c2, B, device=dev)
    for k in range(4):
        x, qn, qr = (t.to(dev) for t in synthetic.draw_chunk(c2, B, 40 + k))
        f0 = l2.frames_written
        V.compress_append(c2, x, w2, l2)
        V.latent_attention(c2, V.absorb_q(c2, qn, qr, wuk2, f0), l2, f0, want_lse=True)
        V.latent_attention_fused(c2, qn, qr, wuk2, wuv2, l2, f0, want_lse=True)
    assert status(f"key-split d_c {d_c}") == 0
cw, bw = WAN, 4
ww = synthetic.draw_weights(cw, 6)[0].to(dev)
lw = V.LatentCache(cw, bw, device=dev)
xw = [synthetic.draw_chunk(cw, bw, 50 + k)[0].to(dev) for k in range(2)]
for k in range(7):                       # 7 chunks of 3 frames fill the 21-frame ring to its last row
    V.compress_append(cw, xw[k % 2], ww, lw)
assert status("paired compress") == 0
# extents one 32-column chunk short: the stores at the ends are reported, codes 90 + site
V.LIB.vmla_debug_shrink_extents(64)
x, qn, qr = (t.to(dev) for t in synthetic.draw_chunk(cfg, B, 30))
f0 = lc.frames_written
assert (f0 % cfg.window_frames) + cfg.chunk_frames > cfg.window_frames - 1   # this chunk fills the last slot
V.compress_append(cfg, x, w, lc)
code_c = status("shrunk compress")
V.latent_attention_fused(cfg, qn, qr, wuk, wuv, lc, f0)
code_a = status("shrunk fused attention")
lw.struct.frames_written = 18            # the paired compress rewrites the ring's last chunk
V.compress_append(cw, xw[0], ww, lw)
code_p = status("shrunk paired compress")
V.LIB.vmla_debug_shrink_extents(0)
V.latent_attention_fused(cfg, qn, qr, wuk, wuv, lc, f0)
assert status("restored") == 0
print("CODES", code_c, code_a, code_p)
"""


def test_checked_build_finds_no_store_outside_its_buffer():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    # incremental: recompiles only what changed since the in-tree checked library was built
    from rank_latent_kv_vmla_b200 import build
    build.build(checked=True)
    env = dict(os.environ, VMLA_LIBRARY=LIB)
    r = subprocess.run([sys.executable, "-c", "ROOT = %r\n" % ROOT + SCRIPT], env=env, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    codes = [l for l in r.stdout.splitlines() if l.startswith("CODES")][0].split()[1:]
    code_c, code_a, code_p = int(codes[0]), int(codes[1]), int(codes[2])
    assert code_c in (91, 92), r.stdout          # c or k_r plane of the newest chunk's last slot
    assert code_a == 99, r.stdout                # the fused kernel's last output chunk
    assert code_p in (91, 92), r.stdout          # the paired compress, same sites
