"""One feed-forward block for the GPU tests: Hid = BF16(GELU(up(X))), Y = down(Hid).

The inputs are seeded and synthetic (the up-projection's activations with outlier
channels, both weights with outlier columns); the GPU side runs dq_ffn_forward
through the C ABI and reads back Hid, Y and the down-projection's workspace; the
checks compare them with the oracle: Hid against GELU of the oracle's up-projection
rows (the Y tolerance carried through GELU plus one BF16 ulp), and the
down-projection, taken on the GPU's own Hid, bit for bit in every quantised tensor
(the cube means too) and within the Y tolerance in its output."""
import numpy as np

import oracle
import synth
from dq_case import assert_y_close, bf16_bits_to_f64, compare_quantised, sfa_unpermute, y_tolerance


def h_tolerance(y_ref: np.ndarray, h_ref: np.ndarray) -> np.ndarray:
    """Tolerance of the BF16 hidden activation: the up-projection's Y tolerance
    through GELU (|GELU'| < 1.13 everywhere) plus one BF16 ulp of the hidden value
    (GELU in fp32, one rounding to BF16)."""
    a = np.abs(h_ref)
    ulp = np.where(a > 0, np.exp2(np.floor(np.log2(np.where(a > 0, a, 1.0))) - 7), 2.0 ** -133)
    return 1.13 * y_tolerance(y_ref) + ulp


class FfnCase:
    def __init__(self, name, T, H, W, cube_up, cube_down, Ci, Cf, Co, r_up, r_down, seed=0x0FF0, bias=False,
                 fp8=False, kgroup_down=0):
        grid = (T, max(1, -(-H // 4)), max(1, -(-W // 4)))
        self.up = synth.Workload(name + "_up", T, H, W, Ci, Cf, r_up, tuple(cube_up), grid, (0.01, 50.0),
                                 (0.01, 20.0))
        self.down = synth.Workload(name + "_down", T, H, W, Cf, Co, r_down, tuple(cube_down), grid, (0.0, 1.0),
                                   (0.01, 20.0))
        self.X = synth.activations(self.up, seed=seed)
        self.Wu = synth.weight(self.up, seed=seed)
        self.Wd = synth.weight(self.down, seed=seed + 1)
        self.L1u, self.L2u, _ = oracle.lowrank_factors(self.Wu, r_up)
        self.L1d, self.L2d, _ = oracle.lowrank_factors(self.Wd, r_down)
        # optional linear biases of both layers (BF16 bits)
        self.bu = synth.normal_bf16((Cf,), 0.5, seed, 7) if bias else None
        self.bd = synth.normal_bf16((Co,), 0.5, seed, 8) if bias else None
        # forward options: the FP8 kernel-token product in both layers (restricted-scale weights), and
        # one kernel scale per 64 channels in the down-projection
        self.fp8, self.kgroup_down = fp8, kgroup_down
        self.packed = None

    def fused_expected(self, dq) -> bool:
        u, d = self.up, self.down
        return dq.dq_ffn_fused_statistics(u.T, u.H, u.W, u.cube, d.cube)

    def run_gpu(self, dq, torch, ffn_flags=0, gelu_layer=False):
        """dq_ffn_forward; with gelu_layer also the up-projection alone through
        dq_linear_forward_opts(epilogue=DQ_EPILOGUE_GELU)."""
        u, d = self.up, self.down
        if self.packed is None:
            pf = dq.DQ_PACK_C2 if self.fp8 else 0
            pu, L1mu, L2su, _ = dq.dq_pack_weight_factors(self.Wu, self.L1u, self.L2u, pack_flags=pf)
            pd, L1md, L2sd, S_Wd = dq.dq_pack_weight_factors(self.Wd, self.L1d, self.L2d, pack_flags=pf)
            if self.bu is not None:
                dq.dq_pack_bias(pu, self.bu)
                dq.dq_pack_bias(pd, self.bd)
            self.packed = (pu, L1mu, L2su, pd, L1md, L2sd, S_Wd)
        pu, L1mu, L2su, pd, L1md, L2sd, S_Wd = self.packed
        dev = torch.device("cuda")
        t16 = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(dev)
        Xd = t16(self.X)
        Pu, Pd = torch.from_numpy(pu).to(dev), torch.from_numpy(pd).to(dev)
        L1u, L2u, L1d, L2d = t16(L1mu), t16(L2su), t16(L1md), t16(L2sd)
        Hd = torch.empty((u.N, u.Co), dtype=torch.int16, device=dev)
        Yd = torch.empty((u.N, d.Co), dtype=torch.int16, device=dev)
        kp = dq.DQ_KERNEL_PRODUCT_FP8 if self.fp8 else dq.DQ_KERNEL_PRODUCT_BF16
        ou = dict(kernel_product=kp)
        od = dict(kernel_product=kp, kernel_group=self.kgroup_down)
        lu = dq.dq_workspace_layout_opts(u.T, u.H, u.W, *u.cube, u.Ci, u.Co, u.rank, **ou)
        ld = dq.dq_workspace_layout_opts(d.T, d.H, d.W, *d.cube, d.Ci, d.Co, d.rank, **od)
        wsu = torch.zeros(lu.total_bytes, dtype=torch.uint8, device=dev)
        wsd = torch.zeros(ld.total_bytes, dtype=torch.uint8, device=dev)
        st = torch.cuda.current_stream()
        if self.fp8 or self.kgroup_down:
            dq.dq_ffn_forward_opts(Xd, u.T, u.H, u.W, u.cube, d.cube, u.Ci, u.Co, d.Co, u.rank, d.rank, Pu, L1u, L2u,
                                   Pd, L1d, L2d, Hd, Yd, wsu, lu.total_bytes, wsd, ld.total_bytes, ffn_flags, None, st,
                                   opts_up=ou, opts_down=od)
        else:
            dq.dq_ffn_forward(Xd, u.T, u.H, u.W, u.cube, d.cube, u.Ci, u.Co, d.Co, u.rank, d.rank, Pu, L1u, L2u, Pd,
                              L1d, L2d, Hd, Yd, wsu, lu.total_bytes, wsd, ld.total_bytes, ffn_flags, None, st)
        torch.cuda.synchronize()
        out = dict(status_up=dq.dq_read_device_status(wsu, st, clear=True),
                   status=dq.dq_read_device_status(wsd, st, clear=True),
                   H=Hd.cpu().numpy().view(np.uint16), Y=Yd.cpu().numpy().view(np.uint16))
        if gelu_layer:
            H2 = torch.empty_like(Hd)
            dq.dq_linear_forward_opts(Xd, u.T, u.H, u.W, *u.cube, u.Ci, u.Co, u.rank, Pu, L1u, L2u, H2, wsu,
                                      lu.total_bytes, dq.DQ_STAGE_ALL, None, st, epilogue=dq.DQ_EPILOGUE_GELU, **ou)
            torch.cuda.synchronize()
            assert dq.dq_read_device_status(wsu, st, clear=True) == 0
            out["H_layer"] = H2.cpu().numpy().view(np.uint16)
        w = wsd.cpu().numpy()
        N, K, C = ld.N, ld.K, d.Ci
        kg = self.kgroup_down
        ns8, acols = (C // kg if kg else 1), (2 * C if kg else C)
        out.update(layout=ld, S_W=S_Wd, packed=pd,
                   means=w[ld.off_means:ld.off_means + 4 * K * C].view(np.uint32).reshape(K, C),
                   amax_delta=w[ld.off_scalars:ld.off_scalars + 4].view(np.float32)[0],
                   S_delta=w[ld.off_scalars + 4:ld.off_scalars + 8].view(np.float32)[0],
                   s8=w[ld.off_s8:ld.off_s8 + 4 * K * ns8].view(np.float32).reshape((K, ns8) if kg else (K,)),
                   q8=w[ld.off_q8:ld.off_q8 + K * C].reshape(K, C),
                   q8_bf16=None if self.fp8 else
                   w[ld.off_q8_bf16:ld.off_q8_bf16 + 2 * K * acols].view(np.uint16).reshape(K, acols),
                   dcodes=w[ld.off_dcodes:ld.off_dcodes + N * C // 2].reshape(N, C // 2),
                   dscales=sfa_unpermute(w[ld.off_dscales:], N, C))
        return out

    def check(self, g, rows=None) -> dict:
        """Oracle checks of one run (all rows, or the natural token rows given)."""
        u, d = self.up, self.down
        assert g["status_up"] == 0, g["status_up"]
        rows = np.arange(u.N) if rows is None else rows
        act_u = oracle.quantize_activations(self.X, u.T, u.H, u.W, u.cube)
        wq_u = oracle.quantize_weight(self.Wu, self.L1u, self.L2u, c2=self.fp8)
        y_ref = oracle.output_rows(act_u, wq_u, self.X, self.L1u, self.L2u, rows, bias=self.bu)
        h_ref = oracle.ffn_hidden_rows(act_u, wq_u, self.X, self.L1u, self.L2u, rows, bias=self.bu)
        h = bf16_bits_to_f64(g["H"][rows])
        tol = h_tolerance(y_ref, h_ref)
        err = np.abs(h - h_ref)
        assert np.all(err <= tol), ("hidden", float((err / tol).max()), np.argwhere(err > tol)[:5].tolist())
        # the down-projection on the GPU's own hidden activation
        act_d = oracle.quantize_activations(g["H"], d.T, d.H, d.W, d.cube, kernel_group=self.kgroup_down)
        wq_d = oracle.quantize_weight(self.Wd, self.L1d, self.L2d, c2=self.fp8)
        means = oracle.cube_means(g["H"], d.T, d.H, d.W, d.cube)
        bad = np.argwhere(g["means"] != means.view(np.uint32))
        assert bad.size == 0, ("cube means", bad[:5].tolist())
        compare_quantised(g, act_d, wq_d)
        info = assert_y_close(g["Y"][rows], oracle.output_rows(act_d, wq_d, g["H"], self.L1d, self.L2d, rows,
                                                               bias=self.bd))
        info.update(hidden_max_err_over_tol=float((err / tol).max()))
        return info
