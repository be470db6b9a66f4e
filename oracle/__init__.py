"""fp64 CPU oracle for the KDA forward pass. TEST INFRASTRUCTURE ONLY.

Importable by the tests, the smoke check and the bench's CPU-baseline leg;
never by the product path (the ``gated_delta_rule_156_b200`` package).
"""
