"""CPU oracle for the QLoRA NF4 linear layer — TEST INFRASTRUCTURE ONLY.

Plain, slow, obviously-correct numpy restatements of what the web pages on
QLoRA define: the NormalFloat-4 code points, blockwise absmax quantisation,
double quantisation of the block constants, double dequantisation, and the
LoRA linear layer's forward and backward pass (accumulated in float64).

Only the tests, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The
CUDA library never calls it and shares no code, table or constant generator
with it.

Citations name the page and its section, e.g.
"QLoRA: Efficient Finetuning of Quantized LLMs (intuitivepapers.ai), §NormalFloat".

Parity status: every function here is pinned by ``-m "not gpu"`` tests in
``tests/test_oracle_*.py`` against values the pages print, closed forms,
brute force and independent library routines.
"""
