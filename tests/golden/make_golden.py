"""Writes the hand-derived worked examples under tests/golden/.

The pages print no worked numeric example, so each fixture here is a tiny
case whose answer was derived by hand from the formula it cites; the script
only evaluates those closed forms (no call into the oracle or the library).
Run:  python tests/golden/make_golden.py
"""
import json
import math
import os

HERE = os.path.dirname(os.path.abspath(__file__))
e2 = math.exp(2.0)

zero_order = {
    "cite": "PISA - Atenção Esparsa por Partes para Transformers de Difusão Eficientes, "
            "§2 'Algoritmo Central': o_t = N_t / D_t, zero-order term alpha_{t,j} (sum_n v_{j,n}) "
            "in N_t for unselected blocks, its denominator counterpart B alpha_{t,j}; "
            "SLA2 §2A mixture O = alpha O_s + (1 - alpha) O_l; SALAD §2 ReLU linear branch",
    "derivation": [
        "d=1, block B=2, N=4 (KV blocks 0 and 1), softmax scale s=1, one query block (rows 0,1).",
        "K = [0, 0 | 1, 3], V = [1, 2 | 3, 5], Q = [1, 0]; selected S_0 = {0}, unselected U_0 = {1}.",
        "exact part for q: e^{q*0}*1 + e^{q*0}*2 = 3, denominator 2 (both rows).",
        "block 1: centroid kbar_1 = 2, value sum 8: numerator += e^{2q} * 8, denominator += 2 e^{2q}.",
        "zero_order row q=1: (3 + 8 e^2) / (2 + 2 e^2);  row q=0: (3 + 8) / (2 + 2) = 2.75.",
        "drop: 3/2 = 1.5 for both rows.",
        "linear_mix, alpha = 0.25, eps = 1e-6: O_l(q=1) = (1*3 + 3*5) / (1 + 3 + eps) = 18/(4+eps), "
        "O_l(q=0) = 0 / eps = 0; O = 0.25*1.5 + 0.75*O_l.",
    ],
    "block": 2, "scale": 1.0, "eps": 1e-6,
    "Q": [[1.0], [0.0], [0.0], [0.0]],
    "K": [[0.0], [0.0], [1.0], [3.0]],
    "V": [[1.0], [2.0], [3.0], [5.0]],
    "block_idx": [[0], [1]],
    "alpha": [0.25],
    "expected_rows_0_1": {
        "zero_order": [(3 + 8 * e2) / (2 + 2 * e2), 11.0 / 4.0],
        "drop": [1.5, 1.5],
        "linear_mix": [0.25 * 1.5 + 0.75 * 18.0 / (4.0 + 1e-6), 0.25 * 1.5],
    },
}

taylor2 = {
    "cite": "SPLA - Block Sparse Plus Linear Attention para Modelagem de Contexto Longo, §2.1: "
            "block score exp(q^T kbar)(1 + 1/2 q^T Cov(k) q) with the covariance taken diagonal",
    "derivation": [
        "d=2, block 2, scale 1, pooled query q = [1, 2].",
        "block 0 keys [1,0],[1,2]: mean [1,1], population variance [0,1]: "
        "exp(1+2) * (1 + 0.5*(1*0 + 4*1)) = 3 e^3, log score 3 + ln 3.",
        "block 1 keys [0,0],[2,0]: mean [1,0], variance [1,0]: exp(1) * (1 + 0.5*1) = 1.5 e, "
        "log score 1 + ln 1.5.",
        "dot scores q.kbar: [3, 1]; top-1 = [0].",
    ],
    "qmean": [1.0, 2.0],
    "K": [[1.0, 0.0], [1.0, 2.0], [0.0, 0.0], [2.0, 0.0]],
    "block": 2, "scale": 1.0,
    "expected_log_scores": [3.0 + math.log(3.0), 1.0 + math.log(1.5)],
    "expected_kmean": [[1.0, 1.0], [1.0, 0.0]],
    "expected_kvar": [[0.0, 1.0], [1.0, 0.0]],
    "expected_dot": [3.0, 1.0],
}

for name, obj in (("pisa_zero_order_worked.json", zero_order),
                  ("spla_taylor2_worked.json", taylor2)):
    with open(os.path.join(HERE, name), "w") as f:
        json.dump(obj, f, indent=1)
        f.write("\n")
print("written")
