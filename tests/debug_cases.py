"""Seeded optimizer steps for comparing the release and debug libraries.

Run as a script (``python tests/debug_cases.py OUT.npz``) under the library
that the MA_LIBRARY environment variable selects; it saves every case's
updated weights, momentum or AdamW state, the status word, and which build
ran. tests/test_gpu_debug_build.py runs it once per library and compares.

The cases reach every kernel whose device indexing the debug build guards:
AdamW (vector and scalar paths, bf16 and fp32 gradients), the flat and the
transposing momentum passes, the Gram-space chain (its Q_1 kernel, symmetric
products and a = 0 final apply), the direct chain (Gram, apply, and both
final-apply variants: m >= 2048 takes the deep one), single-CTA head slices,
ragged shapes, a schedule with c != 0, and the fp32 (SIMT) mode.
"""
import sys

import numpy as np
import torch

import adamw_hybrid_optimizer_muon_b200 as ma

# (R, C, heads, precision, coefficient table)
MUON = [
    (512, 1024, 1, 0, None),      # Gram-space chain, flat momentum pass
    (1024, 512, 1, 0, None),      # tall: transposing pass, transposed final store
    (520, 2056, 1, 0, None),      # ragged, Gram-space
    (300, 200, 1, 0, None),       # ragged tall, direct chain
    (384, 384, 1, 0, None),       # square, direct chain, shallow final apply
    (2048, 2048, 1, 0, None),     # square, m >= 2048: deep final apply with the a*X term
    (2048, 2560, 1, 0, None),     # wide, m >= 2048: Gram-space, deep final apply with a = 0
    (1024, 512, 8, 0, None),      # head slices of 128 x 512 (single-CTA tiles)
    (256, 384, 1, 1, None),       # fp32 mode (SIMT kernels, fp32 X)
    (512, 768, 1, 0, ((2.0, -1.5, 0.5),)),  # c != 0: the A^2 product, direct chain
]
ADAMW = [(4099, "bf16", 0), (8192 * 3 + 5, "f32", 0), (1001, "bf16", 1)]  # (numel, grad dtype, view offset)


def run(out_path):
    torch.cuda.set_device(0)
    res = {"debug_build": np.array(int(ma.ma_debug_build()))}
    for k, (R, C, heads, prec, co) in enumerate(MUON):
        r = np.random.default_rng(100 + k)
        kw = {"heads": heads, "precision": prec}
        if co is not None:
            kw["coeffs"] = co
        hp = ma.muon_hparams(**kw)
        W = [torch.from_numpy((r.standard_normal((R, C)) * 0.02).astype(np.float32)).cuda() for _ in range(2)]
        M = [torch.zeros((R, C), device="cuda") for _ in range(2)]
        ws = torch.empty(ma.muon_workspace_bytes(2, R, C, hp), dtype=torch.uint8, device="cuda")
        for _ in range(2):  # two steps: the second starts from a nonzero momentum
            G = [torch.from_numpy((r.standard_normal((R, C)) * 1e-3).astype(np.float32)).cuda().bfloat16()
                 for _ in range(2)]
            ma.muon_step_batched(W, G, M, hp, ws)
        torch.cuda.synchronize()
        res[f"muon{k}_status"] = np.array(ma.ma_device_status())
        for b in range(2):
            res[f"muon{k}_W{b}"] = W[b].cpu().numpy()
            res[f"muon{k}_M{b}"] = M[b].cpu().numpy()
    for k, (numel, gdt, off) in enumerate(ADAMW):
        r = np.random.default_rng(200 + k)
        base = [torch.from_numpy(r.standard_normal(numel + off).astype(np.float32)).cuda() for _ in range(3)]
        p, m, v = (t[off:] for t in base)  # an offset view takes the scalar path
        v.abs_()
        g32 = torch.from_numpy(r.standard_normal(numel + off).astype(np.float32)).cuda()[off:]
        g = g32.bfloat16() if gdt == "bf16" else g32
        ma.adamw_step_fused([p], [g], [m], [v], ma.adamw_hparams(lr=0.01, weight_decay=0.01, step=3))
        torch.cuda.synchronize()
        res[f"adamw{k}_status"] = np.array(ma.ma_device_status())
        for name, t in (("p", p), ("m", m), ("v", v)):
            res[f"adamw{k}_{name}"] = t.cpu().numpy()
    np.savez(out_path, **res)


if __name__ == "__main__":
    run(sys.argv[1])
