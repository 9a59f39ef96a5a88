"""Small calls of every kernel family, run in a child process against the debug build
(OSP_LIBRARY=debug, device-side index checks) by tests/test_gpu_bounds.py.

    python -m tests.bounds_cases <out.pt> [expect_bounds]

Writes the outputs (CPU tensors) to <out.pt>.  With `expect_bounds`, every call must instead end
in OSP_ERR_BOUNDS from osp_check_status (the caller shrinks the checks' limits)."""

import sys

import torch

from spacetime_attention_b200 import ops, synthetic as syn


def calls(dev):
    w = syn.custom("b", 1, 2, 64, (4, 8, 8), 0, (16, 24, 24), skiparse_k=2)
    q, k, v = (t.to(dev) for t in syn.make_qkv(w, 77))
    do = syn.randn_bf16(tuple(q.shape), 81).to(dev)
    kt, vt = syn.randn_bf16((1, 40, 2, 64), 82).to(dev), syn.randn_bf16((1, 40, 2, 64), 83).to(dev)
    # d = 128: outputs leave through the staging tile and TMA stores (d >= 96)
    w2 = syn.custom("b2", 1, 2, 128, (2, 8, 10), 0, (32, 48, 48), skiparse_k=2)
    q2, k2, v2 = (t.to(dev) for t in syn.make_qkv(w2, 78))

    def backward():
        o, lse = ops.attn_forward_train(q, k, v, w.grid, 0)
        return ops.attn_backward(q, k, v, o, do, lse, w.grid, 0)

    def packed_training():   # two samples of 100 and 156 rows: packed forward with lse, backward
        o, lse = ops.attn_packed_train(q, k, v, [0, 100, 256])
        return ops.attn_packed_backward(q, k, v, o, do, lse, [0, 100, 256])

    def skiparse_text_training():   # 64 text rows joined to Group Skip k = 2 sets of 96: forward, backward
        g = (4, 8, 6)
        o, lse = ops.attn_forward_train(q, k, v, g, 64, sparse_k=2, mode=1)
        return ops.attn_backward(q, k, v, o, do, lse, g, 64, sparse_k=2, mode=1)

    def temporal_training():   # the per-set temporal kernels (T <= 64): forward with lse, backward
        o, lse = ops.attn_temporal_train(q, k, v, w.grid, causal=True)
        return ops.attn_temporal_backward(q, k, v, o, do, lse, w.grid, causal=True)

    return {
        "rope": lambda: ops.rope3d(q, k, w.grid, 0, w.split),
        "gather": lambda: ops.skiparse_gather(q, k, v, w.grid, 2, 1, split=w.split),
        "scatter": lambda: ops.skiparse_scatter(q.view(2, 128, 2, 64), w.grid, 2, 0),
        "dense": lambda: ops.attn_full(q, k, v, w.grid, 0),
        "dense_d128": lambda: ops.attn_full(q2, k2, v2, w2.grid, 0),
        "skiparse_d128": lambda: ops.skiparse_attn(q2, k2, v2, w2.grid, 2, 1),
        "skiparse": lambda: ops.skiparse_attn(q, k, v, w.grid, 2, 1),
        "cross": lambda: ops.attn_cross(q, kt, vt, w.grid),
        "temporal": lambda: ops.attn_temporal(q, k, v, w.grid, causal=True),
        "packed": lambda: ops.attn_packed(q, k, v, [0, 100, 256]),
        "backward": backward,
        "temporal_training": temporal_training,
        "packed_training": packed_training,
        "skiparse_text_training": skiparse_text_training,
    }


def main():
    out_path = sys.argv[1]
    expect_bounds = len(sys.argv) > 2 and sys.argv[2] == "expect_bounds"
    assert ops.LIB_PATH.endswith("libosp_debug.so"), ops.LIB_PATH
    dev = torch.device("cuda:0")
    results = {}
    for name, fn in calls(dev).items():
        r = fn()
        try:
            ops.check_status(dev)
            status = 0
        except ops.OspError as e:
            status = e.code
        if expect_bounds:
            assert status == 6, f"{name}: status {status}, expected OSP_ERR_BOUNDS (6)"
        else:
            assert status == 0, f"{name}: status {status}"
            rs = r if isinstance(r, tuple) else (r,)
            results[name] = [t.cpu() for t in rs if t is not None]
    torch.save(results, out_path)
    print("ok", sorted(results) if results else "bounds")


if __name__ == "__main__":
    main()
